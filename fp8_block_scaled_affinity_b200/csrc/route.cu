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
constexpr int kLK = 32;   // k per smem stage

// u[t, i] = fp32(sum_k x[t,k] * E[i,k]) with an FP64 accumulator updated in
// ascending k (each bf16*bf16 product is exact in FP64, so fma == mul+add).
// 256 threads; thread (ty, tx) owns tokens 4ty..4ty+3 and experts 4tx..4tx+3.
__global__ void __launch_bounds__(256) route_logits_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ E, int T, int d, int n_routed,
    float* __restrict__ u) {
    __shared__ __align__(16) double xs[kLK][kLT];
    __shared__ __align__(16) double es[kLK][kLE];
    const int t0 = blockIdx.x * kLT, e0 = blockIdx.y * kLE;
    const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
    const int lrow = tid >> 2, lk = (tid & 3) * 8;
    const bool xrow_ok = t0 + lrow < T, erow_ok = e0 + lrow < n_routed;
    const uint4* xp = reinterpret_cast<const uint4*>(x + int64_t(t0 + lrow) * d + lk);
    const uint4* ep = reinterpret_cast<const uint4*>(E + int64_t(e0 + lrow) * d + lk);
    double acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
    for (int k0 = 0; k0 < d; k0 += kLK) {
        const uint4 xv = xrow_ok ? __ldg(xp + k0 / 8) : make_uint4(0u, 0u, 0u, 0u);
        const uint4 ev = erow_ok ? __ldg(ep + k0 / 8) : make_uint4(0u, 0u, 0u, 0u);
        __syncthreads();
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, ew[4] = {ev.x, ev.y, ev.z, ev.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            xs[lk + 2 * j][lrow] = (double)bf16_lo(xw[j]);
            xs[lk + 2 * j + 1][lrow] = (double)bf16_hi(xw[j]);
            es[lk + 2 * j][lrow] = (double)bf16_lo(ew[j]);
            es[lk + 2 * j + 1][lrow] = (double)bf16_hi(ew[j]);
        }
        __syncthreads();
#pragma unroll 8
        for (int k = 0; k < kLK; ++k) {
            const double2 xa = *reinterpret_cast<const double2*>(&xs[k][ty * 4]);
            const double2 xb = *reinterpret_cast<const double2*>(&xs[k][ty * 4 + 2]);
            const double2 ea = *reinterpret_cast<const double2*>(&es[k][tx * 4]);
            const double2 eb = *reinterpret_cast<const double2*>(&es[k][tx * 4 + 2]);
            const double xv4[4] = {xa.x, xa.y, xb.x, xb.y}, ev4[4] = {ea.x, ea.y, eb.x, eb.y};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fma(xv4[i], ev4[j], acc[i][j]);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = t0 + ty * 4 + i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int e = e0 + tx * 4 + j;
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
    route_logits_kernel<<<g1, 256, 0, st>>>(x, router_w, T, d, N, u);
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
