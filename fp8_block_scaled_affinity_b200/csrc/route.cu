// Token-to-expert routing ("DeepSeek-V3 Technical Report" notes page,
// section "DeepSeekMoE and auxiliary-loss-free load balancing"): sigmoid
// affinity, bias for the routing decision only, group-limited top-K (the
// "at most M nodes" rule with expert groups standing in for nodes), gates
// normalised from the unbiased affinities, and the per-batch expert load
// histogram.  Gating stays in high precision (section "FP8 mixed precision
// training"): the logits are FP64 dot products summed in ascending k, so the
// result is reproducible bit for bit.
#include <math.h>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kLT = 64;   // tokens per logits tile
constexpr int kLE = 64;   // experts per logits tile
constexpr int kLK = 16;   // k per smem stage (double-buffered)
constexpr int kLV = kLK / 8;  // 16-byte vectors per row and stage
constexpr int kLThreads = 64;

// u[t, i] = fp32(sum_k x[t,k] * E[i,k]) with an FP64 accumulator updated in
// ascending k (each bf16*bf16 product is exact in FP64, so fma == mul+add).
// 64 threads; thread (ty, tx) owns tokens 8ty..8ty+7 and experts 8tx..8tx+7
// of the 64 x 64 tile (64 FP64 accumulators).  Shared memory holds the tile's
// K chunk as doubles; the experts are stored interleaved (expert 8tx+j at
// column 8j+tx) so that the 8 threads of a row read consecutive doubles.
// Chunks are double-buffered and the next one is fetched into registers
// while the current one is multiplied.
__global__ void __launch_bounds__(kLThreads) route_logits_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ E, int T, int d, int n_routed,
    float* __restrict__ u) {
    __shared__ __align__(16) double xs[2][kLK][kLT];
    __shared__ __align__(16) double es[2][kLK][kLE];
    const int t0 = blockIdx.x * kLT, e0 = blockIdx.y * kLE;
    const int tid = threadIdx.x, ty = tid >> 3, tx = tid & 7;
    // loader: thread tid stages row tid of the x tile and row tid of the E
    // tile, kLK k values of each per chunk
    const bool xrow_ok = t0 + tid < T, erow_ok = e0 + tid < n_routed;
    const uint4* xp = reinterpret_cast<const uint4*>(x + int64_t(t0 + tid) * d);
    const uint4* ep = reinterpret_cast<const uint4*>(E + int64_t(e0 + tid) * d);
    const int ecol = (tid & 7) * 8 + (tid >> 3);  // interleaved column of expert tid
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    uint4 xv[kLV], ev[kLV];
#pragma unroll
    for (int i = 0; i < kLV; ++i) {
        xv[i] = xrow_ok ? __ldg(xp + i) : zero;
        ev[i] = erow_ok ? __ldg(ep + i) : zero;
    }
    double acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.0;
    int buf = 0;
    for (int k0 = 0; k0 < d; k0 += kLK, buf ^= 1) {
#pragma unroll
        for (int i = 0; i < kLV; ++i) {
            const uint32_t xw[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
            const uint32_t ew[4] = {ev[i].x, ev[i].y, ev[i].z, ev[i].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int kk = 8 * i + 2 * j;
                xs[buf][kk][tid] = (double)bf16_lo(xw[j]);
                xs[buf][kk + 1][tid] = (double)bf16_hi(xw[j]);
                es[buf][kk][ecol] = (double)bf16_lo(ew[j]);
                es[buf][kk + 1][ecol] = (double)bf16_hi(ew[j]);
            }
        }
        __syncthreads();  // this chunk is staged; the other buffer is free again
        if (k0 + kLK < d) {
            const int v = (k0 + kLK) / 8;
#pragma unroll
            for (int i = 0; i < kLV; ++i) {
                xv[i] = xrow_ok ? __ldg(xp + v + i) : zero;
                ev[i] = erow_ok ? __ldg(ep + v + i) : zero;
            }
        }
#pragma unroll 4
        for (int k = 0; k < kLK; ++k) {
            double xr[8], er[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const double2 v2 = *reinterpret_cast<const double2*>(&xs[buf][k][ty * 8 + 2 * i]);
                xr[2 * i] = v2.x;
                xr[2 * i + 1] = v2.y;
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) er[j] = es[buf][k][8 * j + tx];
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fma(xr[i], er[j], acc[i][j]);
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int t = t0 + ty * 8 + i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = e0 + tx * 8 + j;
            if (e < n_routed) u[int64_t(t) * n_routed + e] = __double2float_rn(acc[i][j]);
        }
    }
}

// (value, index) pair order of the selection: larger value first, then the
// lower index.  Invalid entries carry index INT_MAX and lose to valid ones.
__device__ __forceinline__ bool better(float va, int ia, float vb, int ib) {
    if (ib == INT_MAX) return ia != INT_MAX;
    if (ia == INT_MAX) return false;
    return va > vb || (va == vb && ia < ib);
}

__device__ __forceinline__ void warp_argmax(float& v, int& i) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, v, o);
        const int oi = __shfl_xor_sync(0xffffffffu, i, o);
        if (better(ov, oi, v, i)) {
            v = ov;
            i = oi;
        }
    }
}

constexpr int kSelWarps = 8;

// One warp per token.  Shared memory: the block histogram [N_r] followed by
// per-warp s and s' arrays [2][N_r].
__global__ void __launch_bounds__(kSelWarps * 32) route_select_kernel(
    const float* __restrict__ u, int T, int n_routed, int n_groups, int topk_groups, int topk,
    const float* __restrict__ bias, const float* __restrict__ logit_offset,
    int32_t* __restrict__ topk_idx, float* __restrict__ topk_gate,
    int32_t* __restrict__ counts) {
    extern __shared__ __align__(16) float sel_smem[];
    int* hist = reinterpret_cast<int*>(sel_smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float* s = sel_smem + n_routed + warp * 2 * n_routed;
    float* sb = s + n_routed;
    for (int i = threadIdx.x; i < n_routed; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const int t = blockIdx.x * kSelWarps + warp;
    if (t < T) {
        const float* ut = u + int64_t(t) * n_routed;
        for (int i = lane; i < n_routed; i += 32) {
            float ui = ut[i];
            if (logit_offset) ui = __fadd_rn(ui, logit_offset[i]);
            const float si = __double2float_rn(1.0 / (1.0 + exp(-(double)ui)));
            s[i] = si;
            sb[i] = __fadd_rn(si, bias[i]);
        }
        __syncwarp();
        // group scores: lane g holds max s' of group g
        const int ng = n_routed / n_groups;
        float gv = 0.0f;
        int gi = INT_MAX;
        if (lane < n_groups) {
            gv = sb[lane * ng];
            for (int j = 1; j < ng; ++j) {
                const float v = sb[lane * ng + j];
                if (v > gv) gv = v;
            }
            gi = lane;
        }
        uint32_t gmask = 0;
        for (int r = 0; r < topk_groups; ++r) {
            float bv = gv;
            int bi = gi;
            warp_argmax(bv, bi);
            gmask |= 1u << bi;
            if (lane == bi) gi = INT_MAX;  // taken
        }
        // top-K experts inside the chosen groups; lane owns experts lane + 32j
        uint32_t taken = 0;
        int my_idx = 0;
        for (int r = 0; r < topk; ++r) {
            float bv = 0.0f;
            int bi = INT_MAX;
            for (int j = 0, i = lane; i < n_routed; ++j, i += 32) {
                if ((taken >> j) & 1u) continue;
                if (!((gmask >> (i / ng)) & 1u)) continue;
                const float v = sb[i];
                if (better(v, i, bv, bi)) {
                    bv = v;
                    bi = i;
                }
            }
            warp_argmax(bv, bi);
            if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
            if (lane == r) my_idx = bi;
        }
        // gates: S = FP64 sum of the chosen unbiased s in slot order
        const float sv = (lane < topk) ? s[my_idx] : 0.0f;
        double S = 0.0;
        for (int r = 0; r < topk; ++r) S += (double)__shfl_sync(0xffffffffu, sv, r);
        if (lane < topk) {
            topk_idx[int64_t(t) * topk + lane] = my_idx;
            topk_gate[int64_t(t) * topk + lane] = __double2float_rn((double)sv / S);
            atomicAdd(&hist[my_idx], 1);
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < n_routed; i += blockDim.x)
        if (hist[i]) atomicAdd(&counts[i], hist[i]);
}

}  // namespace

int validate_shape(const MoeShape* s) {
    if (!s) return MOE_ERR_NULL;
    if (s->T < 0 || s->d <= 0 || s->d % 128 || s->inter <= 0 || s->inter % 128)
        return MOE_ERR_SHAPE;
    if (s->n_routed < 1 || s->n_routed > 1024) return MOE_ERR_SHAPE;
    if (s->n_groups < 1 || s->n_groups > 32 || s->n_routed % s->n_groups) return MOE_ERR_ROUTE;
    if (s->topk_groups < 1 || s->topk_groups > s->n_groups) return MOE_ERR_ROUTE;
    if (s->topk < 1 || s->topk > 32) return MOE_ERR_ROUTE;
    if (int64_t(s->topk_groups) * (s->n_routed / s->n_groups) < s->topk) return MOE_ERR_ROUTE;
    if (int64_t(s->T) * (s->topk + 1) > INT32_MAX) return MOE_ERR_SHAPE;
    return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" MOE_API size_t moe_route_workspace_size(const MoeShape* shape) {
    if (validate_shape(shape) != MOE_OK) return 0;
    return align_up(size_t(shape->T) * shape->n_routed * sizeof(float), 256);
}

extern "C" MOE_API int moe_route(const MoeShape* shape, const uint16_t* x,
                                 const uint16_t* router_w, const float* bias,
                                 const float* logit_offset, int32_t* topk_idx, float* topk_gate,
                                 int32_t* expert_counts, void* ws, size_t ws_bytes,
                                 int* dev_status, void* stream) {
    (void)dev_status;
    int rc = validate_shape(shape);
    if (rc != MOE_OK) return rc;
    if (!router_w || !bias || !expert_counts) return MOE_ERR_NULL;
    const int T = shape->T, d = shape->d, N = shape->n_routed;
    cudaStream_t st = as_stream(stream);
    if (cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * N, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (T == 0) return check_launch();
    if (!x || !topk_idx || !topk_gate) return MOE_ERR_NULL;
    if (!aligned16(x) || !aligned16(router_w)) return MOE_ERR_ALIGN;
    if (!ws || ws_bytes < moe_route_workspace_size(shape)) return MOE_ERR_WORKSPACE;
    float* u = static_cast<float*>(ws);
    dim3 g1((T + kLT - 1) / kLT, (N + kLE - 1) / kLE);
    route_logits_kernel<<<g1, kLThreads, 0, st>>>(x, router_w, T, d, N, u);
    if ((rc = check_launch()) != MOE_OK) return rc;
    const size_t smem = sizeof(float) * size_t(N) * (1 + 2 * kSelWarps);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(route_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(smem)) != cudaSuccess)
        return MOE_ERR_CUDA;
    route_select_kernel<<<(T + kSelWarps - 1) / kSelWarps, kSelWarps * 32, smem, st>>>(
        u, T, N, shape->n_groups, shape->topk_groups, shape->topk, bias, logit_offset, topk_idx,
        topk_gate, expert_counts);
    return check_launch();
}
