// Backward pass of the MoE layer with respect to x and the router weights
// ("DeepSeek-V3 Technical Report" notes page, section "FP8 mixed precision
// training": the Dgrad GEMMs take FP8 operands with fine-grained scales,
// gating stays in high precision; section "DeepSeekMoE and
// auxiliary-loss-free load balancing": gates are the normalised unbiased
// affinities of the chosen experts, the bias only selects, so no gradient
// flows through the choice or the bias).
//
// For an upstream gradient dy of y:
//   1. moe_combine_backward_quant: do = g_k dy (fp32 product) for each
//      routed row, dy for the shared row, quantised in 1x128 tiles along d
//      (the forward's activation rule) into the permuted row order;
//   2. dh = do W2 (grouped FP8 GEMM on the transposed W2, k = d);
//   3. a, c recomputed (grouped GEMM on W13 with fp32 output, k = d);
//   4. moe_swiglu_backward_quant: da = dh c silu'(a), dc = dh silu(a),
//      [da | dc] quantised in 1x128 tiles along 2I;
//   5. dx rows = [da | dc] [W1; W3] (grouped FP8 GEMM on the transposed W13,
//      k = 2I);
//   6. moe_gate_backward: dg_k = <dy, o_k>, dL/ds_j = (dg_j - sum_k g_k dg_k)
//      / S over the chosen experts, dL/du_j = dL/ds_j s_j (1 - s_j) (FP64);
//   7. moe_router_backward: dx_router[t] = sum_k du_tk E[e_k] and
//      dE[e] = sum over the expert's tokens of du x (fp32, fixed order);
//   8. moe_dx_combine: dx[t] = shared row + routed rows + dx_router[t].
// fp8_transpose_w_128x128 gives the transposed weights: a 128x128 block's
// codes move and its scale stays, so the transposed matrix holds the same
// values (the transposed-GEMM need the pages raise in their discussion).
#include <algorithm>

#include "common.cuh"

namespace moe {
namespace {

int warp_blocks(int64_t units) {
    const int64_t cap = int64_t(sm_count()) * 8;
    return int(std::max<int64_t>(1, std::min<int64_t>((units + 7) / 8, cap)));
}

// ------------------------------------------- 1. do rows, quantised 1x128
// A warp per (token, piece of 2P tiles): dy read once in bf16; for every
// destination row the values g * dy (fp32) are quantised with the forward's
// rule (a half-warp per 1x128 tile) and written to that row.
template <int PC>
__global__ void __launch_bounds__(256) combine_backward_quant_kernel(
    const uint4* __restrict__ dy, int T, int d, int K, const int32_t* __restrict__ row_of_pair,
    const float* __restrict__ gate, int64_t rows_total, uint2* __restrict__ dq,
    float* __restrict__ ds) {
    const int lane = threadIdx.x & 31;
    const int nvec = d / 8, nkb = d / 128;
    const int pieces = (nvec + 32 * PC - 1) / (32 * PC);
    const int64_t units = int64_t(T) * pieces;
    const int64_t warps_total = int64_t(gridDim.x) * (blockDim.x / 32);
    for (int64_t un = int64_t(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5); un < units;
         un += warps_total) {
        const int t = int(un / pieces);
        const int c0 = int(un - int64_t(t) * pieces) * (32 * PC);
        int my_row = 0;
        float my_g = 1.0f;
        if (lane < K) {
            my_row = row_of_pair[int64_t(t) * K + lane];
            my_g = gate[int64_t(t) * K + lane];
        }
        uint4 v[PC];
#pragma unroll
        for (int j = 0; j < PC; ++j) {
            const int c = c0 + lane + 32 * j;
            v[j] = c < nvec ? __ldg(dy + int64_t(t) * nvec + c) : make_uint4(0u, 0u, 0u, 0u);
        }
        // each tile's max |dy| once: for g >= 0, max |fp32(g v)| over a tile
        // is fp32(g max |v|) (rounding is monotone), so every row's scale
        // follows from it without another reduction
        float tmax[PC];
#pragma unroll
        for (int j = 0; j < PC; ++j) {
            const uint4 w = v[j];
            float a = fmaxf(fmaxf(fabsf(bf16_lo(w.x)), fabsf(bf16_hi(w.x))),
                            fmaxf(fabsf(bf16_lo(w.y)), fabsf(bf16_hi(w.y))));
            a = fmaxf(a, fmaxf(fmaxf(fabsf(bf16_lo(w.z)), fabsf(bf16_hi(w.z))),
                               fmaxf(fabsf(bf16_lo(w.w)), fabsf(bf16_hi(w.w)))));
#pragma unroll
            for (int o = 8; o >= 1; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
            tmax[j] = a;
        }
        const int tile = c0 / 16 + lane;
        for (int k = 0; k <= K; ++k) {
            const int row = k < K ? __shfl_sync(0xffffffffu, my_row, k) : T * K + t;
            const float g = k < K ? __shfl_sync(0xffffffffu, my_g, k) : 1.0f;
            if (row < 0) continue;
            float tile_scale = 1.0f;
#pragma unroll
            for (int j = 0; j < PC; ++j) {
                const uint4 w = v[j];
                float scale, inv;
                scale_from_amax(__fmul_rn(fabsf(g), tmax[j]), scale, inv);
                const float f[8] = {__fmul_rn(g, bf16_lo(w.x)), __fmul_rn(g, bf16_hi(w.x)),
                                    __fmul_rn(g, bf16_lo(w.y)), __fmul_rn(g, bf16_hi(w.y)),
                                    __fmul_rn(g, bf16_lo(w.z)), __fmul_rn(g, bf16_hi(w.z)),
                                    __fmul_rn(g, bf16_lo(w.w)), __fmul_rn(g, bf16_hi(w.w))};
                const uint32_t a0 = e4m3x2(__fmul_rn(f[0], inv), __fmul_rn(f[1], inv));
                const uint32_t a1 = e4m3x2(__fmul_rn(f[2], inv), __fmul_rn(f[3], inv));
                const uint32_t a2 = e4m3x2(__fmul_rn(f[4], inv), __fmul_rn(f[5], inv));
                const uint32_t a3 = e4m3x2(__fmul_rn(f[6], inv), __fmul_rn(f[7], inv));
                const int c = c0 + lane + 32 * j;
                if (c < nvec) dq[int64_t(row) * nvec + c] = make_uint2(a0 | (a1 << 16), a2 | (a3 << 16));
                const float sj = __shfl_sync(0xffffffffu, scale, (lane & 1) * 16);
                if ((lane >> 1) == j) tile_scale = sj;
            }
            if (lane < 2 * PC && tile < nkb) ds[int64_t(tile) * rows_total + row] = tile_scale;
        }
    }
}

// ------------------------------------------- 4. SwiGLU backward, quantised
// sigmoid with the fast exponential and a correctly rounded reciprocal (a few
// ulps, as in the forward SwiGLU epilogue; e^-a = inf gives 0)
__device__ __forceinline__ float fast_sigmoid(float a) { return __frcp_rn(1.0f + __expf(-a)); }

// A warp per (row, piece of 2P tiles of the 2I-wide row [da | dc]).
template <int PC>
__global__ void __launch_bounds__(256) swiglu_backward_quant_kernel(
    const float* __restrict__ dh, const float* __restrict__ ac, int64_t rows, int I,
    int64_t rows_total, uint2* __restrict__ q, float* __restrict__ qs) {
    const int lane = threadIdx.x & 31;
    const int n2 = 2 * I;
    const int nvec = n2 / 8, nkb = n2 / 128;
    const int pieces = (nvec + 32 * PC - 1) / (32 * PC);
    const int64_t units = rows * pieces;
    const int64_t warps_total = int64_t(gridDim.x) * (blockDim.x / 32);
    for (int64_t un = int64_t(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5); un < units;
         un += warps_total) {
        const int64_t r = un / pieces;
        const int c0 = int(un - r * pieces) * (32 * PC);
        const float* dhr = dh + r * I;
        const float* ar = ac + r * n2;
        float tile_scale = 1.0f;
#pragma unroll
        for (int j = 0; j < PC; ++j) {
            const int c = c0 + lane + 32 * j;  // vector of 8 values of [da | dc]
            float f[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (c < nvec) {
                const int col = 8 * c;
                const bool is_da = col < I;
                const int feat = is_da ? col : col - I;
                const float4 h0 = *reinterpret_cast<const float4*>(dhr + feat);
                const float4 h1 = *reinterpret_cast<const float4*>(dhr + feat + 4);
                const float4 a0 = *reinterpret_cast<const float4*>(ar + feat);
                const float4 a1 = *reinterpret_cast<const float4*>(ar + feat + 4);
                const float hv[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
                const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                float cv[8];
                if (is_da) {
                    const float4 u0 = *reinterpret_cast<const float4*>(ar + I + feat);
                    const float4 u1 = *reinterpret_cast<const float4*>(ar + I + feat + 4);
                    cv[0] = u0.x; cv[1] = u0.y; cv[2] = u0.z; cv[3] = u0.w;
                    cv[4] = u1.x; cv[5] = u1.y; cv[6] = u1.z; cv[7] = u1.w;
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float a = av[i];
                    const float sg = fast_sigmoid(a);
                    f[i] = is_da ? hv[i] * cv[i] * sg * (1.0f + a * (1.0f - sg)) : hv[i] * a * sg;
                }
            }
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
            for (int o = 8; o >= 1; o >>= 1)
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            float scale, inv;
            scale_from_amax(amax, scale, inv);
            const uint32_t b0 = e4m3x2(__fmul_rn(f[0], inv), __fmul_rn(f[1], inv));
            const uint32_t b1 = e4m3x2(__fmul_rn(f[2], inv), __fmul_rn(f[3], inv));
            const uint32_t b2 = e4m3x2(__fmul_rn(f[4], inv), __fmul_rn(f[5], inv));
            const uint32_t b3 = e4m3x2(__fmul_rn(f[6], inv), __fmul_rn(f[7], inv));
            if (c < nvec) q[r * nvec + c] = make_uint2(b0 | (b1 << 16), b2 | (b3 << 16));
            const float sj = __shfl_sync(0xffffffffu, scale, (lane & 1) * 16);
            if ((lane >> 1) == j) tile_scale = sj;
        }
        const int tile = c0 / 16 + lane;
        if (lane < 2 * PC && tile < nkb) qs[int64_t(tile) * rows_total + r] = tile_scale;
    }
}

// ------------------------------------------- 6. gate gradients (FP64)
// A warp per token: dg_k = <dy, o_k> summed in FP64.  A lane takes four
// consecutive values per step (one 8-byte load of dy, one 16-byte load of
// each of the KM rows, all in flight together) and keeps KM FP64 partial
// sums; one shuffle tree per slot at the end.  Then the chosen scores'
// gradients in FP64.
template <int KM>
__global__ void __launch_bounds__(256) gate_backward_kernel(
    const uint16_t* __restrict__ dy, const float* __restrict__ o, int T, int d, int K,
    const int32_t* __restrict__ row_of_pair, const float* __restrict__ score,
    float* __restrict__ dgate, float* __restrict__ du) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (t >= T) return;
    const float4* rows[KM];
    double acc[KM];
#pragma unroll
    for (int k = 0; k < KM; ++k) {
        const int row = k < K ? row_of_pair[int64_t(t) * K + k] : -1;
        rows[k] = row >= 0 ? reinterpret_cast<const float4*>(o + int64_t(row) * d) : nullptr;
        acc[k] = 0.0;
    }
    const uint2* dyr = reinterpret_cast<const uint2*>(dy + int64_t(t) * d);
    for (int c = lane; c < d / 4; c += 32) {
        const uint2 w = __ldg(dyr + c);
        const double y0 = bf16_lo(w.x), y1 = bf16_hi(w.x), y2 = bf16_lo(w.y), y3 = bf16_hi(w.y);
        float4 v[KM];
#pragma unroll
        for (int k = 0; k < KM; ++k)
            v[k] = rows[k] ? __ldg(rows[k] + c) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int k = 0; k < KM; ++k)
            acc[k] += y0 * double(v[k].x) + y1 * double(v[k].y) + y2 * double(v[k].z) +
                      y3 * double(v[k].w);
    }
    double my_dg = 0.0;
#pragma unroll
    for (int k = 0; k < KM; ++k) {
        double a = acc[k];
#pragma unroll
        for (int s2 = 16; s2 >= 1; s2 >>= 1) a += __shfl_xor_sync(0xffffffffu, a, s2);
        if (lane == k) my_dg = a;
    }
    const double s = lane < K ? double(score[int64_t(t) * K + lane]) : 0.0;
    double S = s;
#pragma unroll
    for (int o2 = 16; o2 >= 1; o2 >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o2);
    double term = lane < K ? (s / S) * my_dg : 0.0;
#pragma unroll
    for (int o2 = 16; o2 >= 1; o2 >>= 1) term += __shfl_xor_sync(0xffffffffu, term, o2);
    if (lane < K) {
        const double ds = (my_dg - term) / S;
        dgate[int64_t(t) * K + lane] = float(my_dg);
        du[int64_t(t) * K + lane] = float(ds * s * (1.0 - s));
    }
}

// ------------------------------------------- 7. router gradients
// dx_router: a warp per (token, 64-float4 slice), the K chosen router rows
// weighted by du in slot order.
__global__ void __launch_bounds__(256) router_dx_kernel(
    const uint16_t* __restrict__ E, const float* __restrict__ du,
    const int32_t* __restrict__ topk_idx, int T, int d, int K, int n_routed,
    float* __restrict__ dx, int* dev_status) {
    const int lane = threadIdx.x & 31;
    const int chunks = (d + 255) / 256;  // 256 values (8 per lane) per unit
    const int64_t units = int64_t(T) * chunks;
    const int64_t warps_total = int64_t(gridDim.x) * (blockDim.x / 32);
    for (int64_t u = int64_t(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5); u < units;
         u += warps_total) {
        const int64_t t = u / chunks;
        const int c = int(u - t * chunks) * 256 + lane * 8;
        if (c >= d) continue;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int k = 0; k < K; ++k) {
            const int e = topk_idx[t * K + k];
            if (e < 0 || e >= n_routed) {
                set_status(dev_status, MOE_DEV_BAD_INPUT);
                continue;
            }
            const float g = du[t * K + k];
            const uint4 w = *reinterpret_cast<const uint4*>(E + int64_t(e) * d + c);
            const float ev[8] = {bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y),
                                 bf16_lo(w.z), bf16_hi(w.z), bf16_lo(w.w), bf16_hi(w.w)};
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = __fmaf_rn(g, ev[i], acc[i]);
        }
        float4* out = reinterpret_cast<float4*>(dx + t * d + c);
        out[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        out[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
}

// pair_of_row[row] = t*K + k for each routed row (the permutation's inverse)
__global__ void pair_of_row_kernel(const int32_t* __restrict__ row_of_pair, int64_t pairs,
                                   int64_t routed_rows, int32_t* __restrict__ pair_of_row) {
    const int64_t p = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (p >= pairs) return;
    const int r = row_of_pair[p];
    if (r >= 0 && r < routed_rows) pair_of_row[r] = int32_t(p);
}

// dE in two phases over the experts' 128-row blocks (the layout of the
// weight-gradient operands): a warp per (block, 256-value slice) sums its
// rows in order into a partial row, then a warp per (expert, slice) adds its
// blocks' partials in order.  Every expert's rows are summed in the same
// fixed order whatever the launch shape (deterministic); the hot expert of a
// skewed batch is spread over as many warps as it has blocks.
__global__ void __launch_bounds__(256) router_dE_partial_kernel(
    const uint16_t* __restrict__ x, const float* __restrict__ du,
    const int2* __restrict__ blocks, int n_blocks, const int32_t* __restrict__ pair_of_row, int d,
    int K, float* __restrict__ partial) {
    const int lane = threadIdx.x & 31;
    const int chunks = (d + 255) / 256;
    const int64_t units = int64_t(n_blocks) * chunks;
    const int64_t warps_total = int64_t(gridDim.x) * (blockDim.x / 32);
    for (int64_t u = int64_t(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5); u < units;
         u += warps_total) {
        const int b = int(u / chunks);
        const int c = int(u - int64_t(b) * chunks) * 256 + lane * 8;
        const int2 blk = blocks[b];
        if (blk.y <= 0 || c >= d) continue;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int r = blk.x; r < blk.x + blk.y; ++r) {
            const int p = pair_of_row[r];
            const int t = p / K;
            const float g = du[p];
            const uint4 w = *reinterpret_cast<const uint4*>(x + int64_t(t) * d + c);
            const float xv[8] = {bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y),
                                 bf16_lo(w.z), bf16_hi(w.z), bf16_lo(w.w), bf16_hi(w.w)};
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = __fmaf_rn(g, xv[i], acc[i]);
        }
        float4* out = reinterpret_cast<float4*>(partial + int64_t(b) * d + c);
        out[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        out[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
}

__global__ void __launch_bounds__(256) router_dE_reduce_kernel(
    const float* __restrict__ partial, const int32_t* __restrict__ kb_offsets, int n_routed,
    int d, float* __restrict__ dE) {
    const int lane = threadIdx.x & 31;
    const int chunks = (d + 127) / 128;
    const int64_t units = int64_t(n_routed) * chunks;
    const int64_t warps_total = int64_t(gridDim.x) * (blockDim.x / 32);
    for (int64_t u = int64_t(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5); u < units;
         u += warps_total) {
        const int e = int(u / chunks);
        const int c = int(u - int64_t(e) * chunks) * 128 + lane * 4;
        if (c >= d) continue;
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int b = kb_offsets[e]; b < kb_offsets[e + 1]; ++b) {
            const float4 v = *reinterpret_cast<const float4*>(partial + int64_t(b) * d + c);
            a.x = __fadd_rn(a.x, v.x);
            a.y = __fadd_rn(a.y, v.y);
            a.z = __fadd_rn(a.z, v.z);
            a.w = __fadd_rn(a.w, v.w);
        }
        *reinterpret_cast<float4*>(dE + int64_t(e) * d + c) = a;
    }
}

// ------------------------------------------- 8. dx
__global__ void __launch_bounds__(256) dx_combine_kernel(
    const float4* __restrict__ dx_rows, const float4* __restrict__ dx_router, int T, int d,
    int K, const int32_t* __restrict__ row_of_pair, float4* __restrict__ dx) {
    const int lane = threadIdx.x & 31;
    const int nv = d / 4;
    const int chunks = (nv + 63) / 64;
    const int64_t units = int64_t(T) * chunks;
    const int64_t warps_total = int64_t(gridDim.x) * (blockDim.x / 32);
    for (int64_t u = int64_t(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5); u < units;
         u += warps_total) {
        const int64_t t = u / chunks;
        int my_row = -1;
        if (lane < K) my_row = row_of_pair[t * K + lane];
        for (int j = 0; j < 2; ++j) {
            const int c = int(u - t * chunks) * 64 + lane + 32 * j;
            if (c >= nv) continue;
            float4 a = dx_rows[(int64_t(T) * K + t) * nv + c];  // the shared expert's row
            for (int k = 0; k < K; ++k) {
                const int row = __shfl_sync(0xffffffffu, my_row, k);
                if (row < 0) continue;
                const float4 v = dx_rows[int64_t(row) * nv + c];
                a.x = __fadd_rn(a.x, v.x);
                a.y = __fadd_rn(a.y, v.y);
                a.z = __fadd_rn(a.z, v.z);
                a.w = __fadd_rn(a.w, v.w);
            }
            if (dx_router) {
                const float4 v = dx_router[t * nv + c];
                a.x = __fadd_rn(a.x, v.x);
                a.y = __fadd_rn(a.y, v.y);
                a.z = __fadd_rn(a.z, v.z);
                a.w = __fadd_rn(a.w, v.w);
            }
            dx[t * nv + c] = a;
        }
    }
}

// ------------------------------------------- transposed weights
// A CTA per 128x128 block: the block's rows read with 16-byte loads into
// shared memory (rows padded to 144 bytes), then each thread gathers 16
// consecutive source rows of one column into one 16-byte store of the
// transposed row.  The block's scale moves to the transposed position.
constexpr int kTPitch = 144;  // bytes per staged row (16-byte aligned, spreads banks)
__global__ void __launch_bounds__(256) transpose_w_kernel(
    const uint8_t* __restrict__ q, const float* __restrict__ s, int64_t mats, int rows,
    int cols, uint8_t* __restrict__ qt, float* __restrict__ st) {
    __shared__ __align__(16) uint8_t tile[128 * kTPitch];
    const int rb = rows / 128, cb = cols / 128;
    const int64_t blocks = mats * rb * cb;
    for (int64_t b = blockIdx.x; b < blocks; b += gridDim.x) {
        const int64_t m = b / (int64_t(rb) * cb);
        const int i = int((b / cb) % rb), j = int(b % cb);
        const uint8_t* src = q + (m * rows + int64_t(i) * 128) * cols + int64_t(j) * 128;
        // 128 rows x 8 vectors of 16 bytes: four per thread
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int e = threadIdx.x + 256 * u;
            const int r = e >> 3, v = e & 7;
            *reinterpret_cast<uint4*>(tile + r * kTPitch + 16 * v) =
                __ldg(reinterpret_cast<const uint4*>(src + int64_t(r) * cols) + v);
        }
        __syncthreads();
        uint8_t* dst = qt + (m * cols + int64_t(j) * 128) * rows + int64_t(i) * 128;
        // output row c (source column c) = 8 vectors of 16 source rows each
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int e = threadIdx.x + 256 * u;
            const int c = e & 127, v = e >> 7;  // consecutive threads: consecutive columns
            uint32_t w[4];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                const uint8_t* col = tile + (16 * v + 4 * q4) * kTPitch + c;
                w[q4] = uint32_t(col[0]) | (uint32_t(col[kTPitch]) << 8) |
                        (uint32_t(col[2 * kTPitch]) << 16) | (uint32_t(col[3 * kTPitch]) << 24);
            }
            *reinterpret_cast<uint4*>(dst + int64_t(c) * rows + 16 * v) =
                make_uint4(w[0], w[1], w[2], w[3]);
        }
        if (threadIdx.x == 0) st[(m * cb + j) * rb + i] = s[(m * rb + i) * cb + j];
        __syncthreads();
    }
}


// ------------------------------------------- weight gradients: 128x1 operands
// K blocks of the weight-gradient GEMMs: each expert's rows (in the
// permutation's order) cut into blocks of 128 from its first row.
// kb_offsets[g] = first block of group g; blocks[b] = (first row, rows).
__global__ void __launch_bounds__(1024) wgrad_layout_kernel(
    const int32_t* __restrict__ row_offsets, int G, int max_blocks, int32_t* __restrict__ kb_offsets,
    int2* __restrict__ blocks, int* dev_status) {
    __shared__ int sums[1024];
    __shared__ int total_s;
    // blocks per group, exclusive scan (G <= 1040: a thread may hold two groups)
    const int t = threadIdx.x;
    int nb[2] = {0, 0};
    for (int j = 0; j < 2; ++j) {
        const int g = 2 * t + j;
        if (g < G) {
            const int rows = row_offsets[g + 1] - row_offsets[g];
            nb[j] = rows > 0 ? (rows + 127) / 128 : 0;
        }
    }
    sums[t] = nb[0] + nb[1];
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {
        const int v = t >= o ? sums[t - o] : 0;
        __syncthreads();
        sums[t] += v;
        __syncthreads();
    }
    int run = sums[t] - nb[0] - nb[1];
    if (t == 1023) total_s = sums[t];
    for (int j = 0; j < 2; ++j) {
        const int g = 2 * t + j;
        if (g < G) kb_offsets[g] = min(run, max_blocks);
        run += nb[j];
    }
    __syncthreads();
    const int total = total_s;
    if (t == 0) {
        kb_offsets[G] = min(total, max_blocks);
        if (total > max_blocks) set_status(dev_status, MOE_DEV_BAD_INPUT);
    }
    // the block table
    for (int g = 0; g < G; ++g) {
        const int r0 = row_offsets[g], rows = row_offsets[g + 1] - r0;
        const int b0 = kb_offsets[g];
        for (int j = t; j * 128 < rows; j += blockDim.x) {
            const int b = b0 + j;
            if (b < max_blocks) blocks[b] = make_int2(r0 + 128 * j, min(128, rows - 128 * j));
        }
    }
    for (int b = total + t; b < max_blocks; b += blockDim.x) blocks[b] = make_int2(0, 0);
}

enum WgSource { kWgX = 0, kWgDo = 1, kWgH = 2, kWgDac = 3 };

struct WgSrc {
    const uint16_t* x;          // x or dy, bf16 [T, d]
    const float* gate;          // [T, K]
    const int32_t* pair_of_row; // [T * K]
    const float* dh;            // [rows, I]
    const float* ac;            // [rows, 2I]
    int T, K, I;
};

// token of a permutation row and the gate its gradient carries
__device__ __forceinline__ int wg_token(const WgSrc& s, int r, float& g) {
    const int TK = s.T * s.K;
    if (r >= TK) {
        g = 1.0f;
        return r - TK;
    }
    const int p = s.pair_of_row[r];
    g = s.gate ? s.gate[p] : 1.0f;
    return p / s.K;
}



// A CTA per (128-row block, 64 output features): the block's values in
// shared memory, one amax per feature over the block's rows, codes written
// transposed (the block's 128 codes of a feature contiguous).
template <int SRC>
__global__ void __launch_bounds__(256) wgrad_quant_kernel(
    WgSrc src, const int2* __restrict__ blocks, int n_blocks, int F, int64_t kpitch,
    uint8_t* __restrict__ qt, float* __restrict__ st) {
    __shared__ __align__(16) float tile[128][68];
    __shared__ float red[4][64];
    __shared__ int tok_s[128];    // gathered sources: token of each row of the block
    __shared__ float gate_s[128]; // and the gate its gradient carries
    const int fchunks = F / 64;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int n_units = n_blocks * fchunks;  // < 2^31 (checked by the launch)
    for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
        const int b = u / fchunks;
        const int f0 = (u - b * fchunks) * 64;
        const int2 blk = blocks[b];
        if (blk.y <= 0) continue;  // past the last expert's rows: never read (uniform)
        if (SRC == kWgX || SRC == kWgDo) {
            // the block's tokens once, not once per lane and row
            if (threadIdx.x < 128) {
                float g = 0.0f;
                tok_s[threadIdx.x] =
                    int(threadIdx.x) < blk.y ? wg_token(src, blk.x + int(threadIdx.x), g) : -1;
                gate_s[threadIdx.x] = g;
            }
            __syncthreads();
        }
        // ---- load: warp w, rows w, w + 8, ...; lane: features f0 + 2 lane, +1.
        // Eight rows at a time: their token indices first, then all their
        // loads, then the arithmetic (a warp keeps eight loads in flight).
        const int fl = f0 + 2 * lane;
        // rows per batch: all 16 of the warp's rows for the gathered bf16
        // sources (their token indices, then their loads, all in flight)
        constexpr int RB = (SRC == kWgX || SRC == kWgDo) ? 16 : 8;
        for (int i0 = 0; i0 < 16; i0 += RB) {
            float v0[RB], v1[RB];
            if (SRC == kWgX || SRC == kWgDo) {
                int tok[RB];
                float g[RB];
#pragma unroll
                for (int i = 0; i < RB; ++i) {
                    const int rr = warp + 8 * (i0 + i);
                    tok[i] = tok_s[rr];
                    g[i] = gate_s[rr];
                }
                uint32_t w2[RB];
#pragma unroll
                for (int i = 0; i < RB; ++i)
                    w2[i] = tok[i] >= 0
                                ? __ldg(reinterpret_cast<const uint32_t*>(src.x + int64_t(tok[i]) * F + fl))
                                : 0u;
#pragma unroll
                for (int i = 0; i < RB; ++i) {
                    v0[i] = bf16_lo(w2[i]);
                    v1[i] = bf16_hi(w2[i]);
                    if (SRC == kWgDo) {
                        v0[i] = __fmul_rn(g[i], v0[i]);
                        v1[i] = __fmul_rn(g[i], v1[i]);
                    }
                }
            } else if (SRC == kWgH) {
                float2 a[8], c[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int rr = warp + 8 * (i0 + i);
                    a[i] = c[i] = make_float2(0.f, 0.f);
                    if (rr < blk.y) {
                        const float* ar = src.ac + int64_t(blk.x + rr) * 2 * src.I;
                        a[i] = __ldg(reinterpret_cast<const float2*>(ar + fl));
                        c[i] = __ldg(reinterpret_cast<const float2*>(ar + src.I + fl));
                    }
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    v0[i] = a[i].x * fast_sigmoid(a[i].x) * c[i].x;
                    v1[i] = a[i].y * fast_sigmoid(a[i].y) * c[i].y;
                }
            } else {  // [da | dc]
                const bool is_da = fl < src.I;
                const int j = is_da ? fl : fl - src.I;
                float2 h[8], a[8], c[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int rr = warp + 8 * (i0 + i);
                    h[i] = a[i] = c[i] = make_float2(0.f, 0.f);
                    if (rr < blk.y) {
                        const int64_t r = blk.x + rr;
                        const float* ar = src.ac + r * 2 * src.I;
                        h[i] = __ldg(reinterpret_cast<const float2*>(src.dh + r * src.I + j));
                        a[i] = __ldg(reinterpret_cast<const float2*>(ar + j));
                        if (is_da) c[i] = __ldg(reinterpret_cast<const float2*>(ar + src.I + j));
                    }
                }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float sg0 = fast_sigmoid(a[i].x), sg1 = fast_sigmoid(a[i].y);
                    if (is_da) {
                        v0[i] = h[i].x * c[i].x * sg0 * (1.0f + a[i].x * (1.0f - sg0));
                        v1[i] = h[i].y * c[i].y * sg1 * (1.0f + a[i].y * (1.0f - sg1));
                    } else {
                        v0[i] = h[i].x * a[i].x * sg0;
                        v1[i] = h[i].y * a[i].y * sg1;
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < RB; ++i)
                *reinterpret_cast<float2*>(&tile[warp + 8 * (i0 + i)][2 * lane]) =
                    make_float2(v0[i], v1[i]);
        }
        __syncthreads();
        // ---- amax per feature, then codes: thread (feature f, quarter q)
        const int f = threadIdx.x & 63, qr = threadIdx.x >> 6;
        float amax = 0.0f;
#pragma unroll 8
        for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(tile[32 * qr + i][f]));
        red[qr][f] = amax;
        __syncthreads();
        amax = fmaxf(fmaxf(red[0][f], red[1][f]), fmaxf(red[2][f], red[3][f]));
        float scale, inv;
        scale_from_amax(amax, scale, inv);
        uint32_t w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float* c = &tile[32 * qr + 4 * i][f];
            const uint32_t lo = e4m3x2(__fmul_rn(c[0], inv), __fmul_rn(c[68], inv));
            const uint32_t hi = e4m3x2(__fmul_rn(c[2 * 68], inv), __fmul_rn(c[3 * 68], inv));
            w[i] = lo | (hi << 16);
        }
        uint4* dst = reinterpret_cast<uint4*>(qt + int64_t(f0 + f) * kpitch + int64_t(b) * 128 +
                                              32 * qr);
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
        if (qr == 0) st[int64_t(b) * F + f0 + f] = scale;
        __syncthreads();
    }
}

// Workspace of moe_router_backward: the routed experts' 128-row blocks and
// one fp32 partial row of dE per block.
struct RouterBwdWs {
    int n_blocks;
    size_t kb_off, blocks, partial, total;
};
RouterBwdWs router_bwd_ws(const MoeShape& s) {
    RouterBwdWs w;
    const int64_t pairs = int64_t(s.T) * s.topk;
    w.n_blocks = int((pairs + 127) / 128 + s.n_routed);
    auto up = [](size_t v) { return (v + 255) / 256 * 256; };
    w.kb_off = 0;
    w.blocks = up(sizeof(int32_t) * (s.n_routed + 1));
    w.partial = w.blocks + up(sizeof(int32_t) * 2 * size_t(w.n_blocks));
    w.total = w.partial + up(sizeof(float) * size_t(w.n_blocks) * s.d);
    return w;
}

int pieces_per(int n, int& PC) {
    const int nkb = n / 128;
    PC = (nkb % 14 == 0 && nkb % 16 != 0) ? 7 : 8;
    return (n / 8 + 32 * PC - 1) / (32 * PC);
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" MOE_API int fp8_transpose_w_128x128(const uint8_t* q, const float* scales,
                                               int64_t mats, int64_t rows, int64_t cols,
                                               uint8_t* qt, float* scales_t, int* dev_status,
                                               void* stream) {
    (void)dev_status;
    if (mats < 0 || rows < 0 || cols < 0 || rows % 128 || cols % 128 || rows > INT32_MAX ||
        cols > INT32_MAX)
        return MOE_ERR_SHAPE;
    if (mats == 0 || rows == 0 || cols == 0) return MOE_OK;
    if (!q || !scales || !qt || !scales_t) return MOE_ERR_NULL;
    if (!aligned16(q) || !aligned16(qt)) return MOE_ERR_ALIGN;
    const int64_t blocks = mats * (rows / 128) * (cols / 128);
    const int grid = int(std::min<int64_t>(blocks, int64_t(sm_count()) * 8));
    transpose_w_kernel<<<grid, 256, 0, as_stream(stream)>>>(q, scales, mats, int(rows), int(cols),
                                                            qt, scales_t);
    return check_launch();
}

extern "C" MOE_API int moe_combine_backward_quant(const MoeShape* shape, const uint16_t* dy,
                                                  const int32_t* row_of_pair,
                                                  const float* topk_gate, uint8_t* do_q,
                                                  float* do_scales, int* dev_status,
                                                  void* stream) {
    (void)dev_status;
    int rc = validate_shape(shape);
    if (rc != MOE_OK) return rc;
    const int T = shape->T, d = shape->d, K = shape->topk;
    if (T == 0) return MOE_OK;
    if (!dy || !row_of_pair || !topk_gate || !do_q || !do_scales) return MOE_ERR_NULL;
    if (!aligned16(dy) || !aligned16(do_q)) return MOE_ERR_ALIGN;
    int PC;
    const int pieces = pieces_per(d, PC);
    const int grid = warp_blocks(int64_t(T) * pieces);
    const int64_t R = int64_t(T) * K + T;
    if (PC == 7)
        combine_backward_quant_kernel<7><<<grid, 256, 0, as_stream(stream)>>>(
            reinterpret_cast<const uint4*>(dy), T, d, K, row_of_pair, topk_gate, R,
            reinterpret_cast<uint2*>(do_q), do_scales);
    else
        combine_backward_quant_kernel<8><<<grid, 256, 0, as_stream(stream)>>>(
            reinterpret_cast<const uint4*>(dy), T, d, K, row_of_pair, topk_gate, R,
            reinterpret_cast<uint2*>(do_q), do_scales);
    return check_launch();
}

extern "C" MOE_API int moe_swiglu_backward_quant(const float* dh, const float* ac, int64_t rows,
                                                 int inter, int64_t rows_total, uint8_t* q,
                                                 float* q_scales, int* dev_status,
                                                 void* stream) {
    (void)dev_status;
    if (rows < 0 || inter <= 0 || inter % 128 || rows_total < rows) return MOE_ERR_SHAPE;
    if (rows == 0) return MOE_OK;
    if (!dh || !ac || !q || !q_scales) return MOE_ERR_NULL;
    if (!aligned16(dh) || !aligned16(ac) || !aligned16(q)) return MOE_ERR_ALIGN;
    int PC;
    const int pieces = pieces_per(2 * inter, PC);
    const int grid = warp_blocks(rows * pieces);
    if (PC == 7)
        swiglu_backward_quant_kernel<7><<<grid, 256, 0, as_stream(stream)>>>(
            dh, ac, rows, inter, rows_total, reinterpret_cast<uint2*>(q), q_scales);
    else
        swiglu_backward_quant_kernel<8><<<grid, 256, 0, as_stream(stream)>>>(
            dh, ac, rows, inter, rows_total, reinterpret_cast<uint2*>(q), q_scales);
    return check_launch();
}

extern "C" MOE_API int moe_gate_backward(const MoeShape* shape, const uint16_t* dy,
                                         const float* expert_out, const int32_t* row_of_pair,
                                         const float* topk_score, float* dgate, float* du,
                                         int* dev_status, void* stream) {
    (void)dev_status;
    int rc = validate_shape(shape);
    if (rc != MOE_OK) return rc;
    const int T = shape->T;
    if (T == 0) return MOE_OK;
    if (!dy || !expert_out || !row_of_pair || !topk_score || !dgate || !du) return MOE_ERR_NULL;
    const int K = shape->topk, grid = (T + 7) / 8;
    cudaStream_t st = as_stream(stream);
    if (!aligned16(expert_out) || (reinterpret_cast<uintptr_t>(dy) & 7)) return MOE_ERR_ALIGN;
    if (K <= 4)
        gate_backward_kernel<4><<<grid, 256, 0, st>>>(dy, expert_out, T, shape->d, K, row_of_pair,
                                                      topk_score, dgate, du);
    else if (K <= 8)
        gate_backward_kernel<8><<<grid, 256, 0, st>>>(dy, expert_out, T, shape->d, K, row_of_pair,
                                                      topk_score, dgate, du);
    else if (K <= 16)
        gate_backward_kernel<16><<<grid, 256, 0, st>>>(dy, expert_out, T, shape->d, K,
                                                       row_of_pair, topk_score, dgate, du);
    else
        gate_backward_kernel<32><<<grid, 256, 0, st>>>(dy, expert_out, T, shape->d, K,
                                                       row_of_pair, topk_score, dgate, du);
    return check_launch();
}

extern "C" MOE_API int moe_router_backward(const MoeShape* shape, const uint16_t* x,
                                           const uint16_t* router_w, const float* du,
                                           const int32_t* topk_idx,
                                           const int32_t* expert_offsets,
                                           const int32_t* row_of_pair, int32_t* pair_scratch,
                                           float* dx_router, float* d_router_w, void* ws,
                                           size_t ws_bytes, int* dev_status, void* stream) {
    int rc = validate_shape(shape);
    if (rc != MOE_OK) return rc;
    const int T = shape->T, d = shape->d, K = shape->topk, N = shape->n_routed;
    if (!d_router_w) return MOE_ERR_NULL;
    cudaStream_t st = as_stream(stream);
    if (T == 0)
        return cudaMemsetAsync(d_router_w, 0, sizeof(float) * N * d, st) == cudaSuccess
                   ? MOE_OK : MOE_ERR_CUDA;
    if (!x || !router_w || !du || !topk_idx || !expert_offsets || !row_of_pair ||
        !pair_scratch || !dx_router || !ws)
        return MOE_ERR_NULL;
    if (!aligned16(x) || !aligned16(router_w) || !aligned16(dx_router) || !aligned16(d_router_w))
        return MOE_ERR_ALIGN;
    const RouterBwdWs W = router_bwd_ws(*shape);
    if (ws_bytes < W.total) return MOE_ERR_WORKSPACE;
    char* base = static_cast<char*>(ws);
    int32_t* kb_off = reinterpret_cast<int32_t*>(base + W.kb_off);
    int2* blocks = reinterpret_cast<int2*>(base + W.blocks);
    float* partial = reinterpret_cast<float*>(base + W.partial);
    const int chunks = (d + 255) / 256;
    router_dx_kernel<<<warp_blocks(int64_t(T) * chunks), 256, 0, st>>>(
        router_w, du, topk_idx, T, d, K, N, dx_router, dev_status);
    if ((rc = check_launch()) != MOE_OK) return rc;
    const int64_t pairs = int64_t(T) * K;
    pair_of_row_kernel<<<int((pairs + 255) / 256), 256, 0, st>>>(row_of_pair, pairs, pairs,
                                                                  pair_scratch);
    if ((rc = check_launch()) != MOE_OK) return rc;
    wgrad_layout_kernel<<<1, 1024, 0, st>>>(expert_offsets, N, W.n_blocks, kb_off, blocks,
                                            dev_status);
    if ((rc = check_launch()) != MOE_OK) return rc;
    router_dE_partial_kernel<<<warp_blocks(int64_t(W.n_blocks) * chunks), 256, 0, st>>>(
        x, du, blocks, W.n_blocks, pair_scratch, d, K, partial);
    if ((rc = check_launch()) != MOE_OK) return rc;
    router_dE_reduce_kernel<<<warp_blocks(int64_t(N) * ((d + 127) / 128)), 256, 0, st>>>(
        partial, kb_off, N, d, d_router_w);
    return check_launch();
}

extern "C" MOE_API size_t moe_router_backward_workspace_size(const MoeShape* shape) {
    if (validate_shape(shape) != MOE_OK) return 0;
    return router_bwd_ws(*shape).total;
}

extern "C" MOE_API int moe_dx_combine(const MoeShape* shape, const float* dx_rows,
                                      const float* dx_router, const int32_t* row_of_pair,
                                      float* dx, int* dev_status, void* stream) {
    (void)dev_status;
    int rc = validate_shape(shape);
    if (rc != MOE_OK) return rc;
    const int T = shape->T;
    if (T == 0) return MOE_OK;
    if (!dx_rows || !row_of_pair || !dx) return MOE_ERR_NULL;
    if (!aligned16(dx_rows) || !aligned16(dx) || (dx_router && !aligned16(dx_router)))
        return MOE_ERR_ALIGN;
    const int chunks = (shape->d / 4 + 63) / 64;
    dx_combine_kernel<<<warp_blocks(int64_t(T) * chunks), 256, 0, as_stream(stream)>>>(
        reinterpret_cast<const float4*>(dx_rows), reinterpret_cast<const float4*>(dx_router), T,
        shape->d, shape->topk, row_of_pair, reinterpret_cast<float4*>(dx));
    return check_launch();
}

extern "C" MOE_API int moe_wgrad_max_blocks(int64_t rows, int n_groups) {
    if (rows < 0 || n_groups < 1) return -1;
    const int64_t b = (rows + 127) / 128 + n_groups;
    return b > INT32_MAX / 128 ? -1 : int(b);
}

extern "C" MOE_API int moe_wgrad_layout(int n_groups, const int32_t* row_offsets,
                                        int max_blocks, int32_t* kb_offsets, int32_t* blocks,
                                        int* dev_status, void* stream) {
    if (n_groups < 1 || n_groups > 2048 || max_blocks < 1) return MOE_ERR_SHAPE;
    if (!row_offsets || !kb_offsets || !blocks) return MOE_ERR_NULL;
    wgrad_layout_kernel<<<1, 1024, 0, as_stream(stream)>>>(row_offsets, n_groups, max_blocks,
                                                           kb_offsets,
                                                           reinterpret_cast<int2*>(blocks),
                                                           dev_status);
    return check_launch();
}

namespace {
template <int SRC>
int launch_wgrad_quant(const WgSrc& src, const int32_t* blocks, int n_blocks, int F,
                       uint8_t* qt, float* st, void* stream) {
    if (n_blocks < 0 || F <= 0 || F % 64) return MOE_ERR_SHAPE;
    if (n_blocks == 0) return MOE_OK;
    if (!blocks || !qt || !st) return MOE_ERR_NULL;
    if (!aligned16(qt)) return MOE_ERR_ALIGN;
    const int64_t units = int64_t(n_blocks) * (F / 64);
    if (units > INT32_MAX) return MOE_ERR_SHAPE;
    const int grid = int(std::min<int64_t>(units, int64_t(sm_count()) * 8));
    wgrad_quant_kernel<SRC><<<grid, 256, 0, as_stream(stream)>>>(
        src, reinterpret_cast<const int2*>(blocks), n_blocks, F, int64_t(n_blocks) * 128, qt, st);
    return check_launch();
}
}  // namespace

extern "C" MOE_API int moe_wgrad_quant_x(const MoeShape* shape, const uint16_t* x,
                                         const int32_t* pair_of_row, const int32_t* blocks,
                                         int n_blocks, uint8_t* xt, float* xt_scales,
                                         int* dev_status, void* stream) {
    (void)dev_status;
    int rc = validate_shape(shape);
    if (rc != MOE_OK) return rc;
    if (shape->T > 0 && (!x || !pair_of_row)) return MOE_ERR_NULL;
    WgSrc s{x, nullptr, pair_of_row, nullptr, nullptr, shape->T, shape->topk, shape->inter};
    return launch_wgrad_quant<kWgX>(s, blocks, n_blocks, shape->d, xt, xt_scales, stream);
}

extern "C" MOE_API int moe_wgrad_quant_do(const MoeShape* shape, const uint16_t* dy,
                                          const float* topk_gate, const int32_t* pair_of_row,
                                          const int32_t* blocks, int n_blocks, uint8_t* dot,
                                          float* dot_scales, int* dev_status, void* stream) {
    (void)dev_status;
    int rc = validate_shape(shape);
    if (rc != MOE_OK) return rc;
    if (shape->T > 0 && (!dy || !topk_gate || !pair_of_row)) return MOE_ERR_NULL;
    WgSrc s{dy, topk_gate, pair_of_row, nullptr, nullptr, shape->T, shape->topk, shape->inter};
    return launch_wgrad_quant<kWgDo>(s, blocks, n_blocks, shape->d, dot, dot_scales, stream);
}

extern "C" MOE_API int moe_wgrad_quant_h(const float* ac, int inter, const int32_t* blocks,
                                         int n_blocks, uint8_t* ht, float* ht_scales,
                                         int* dev_status, void* stream) {
    (void)dev_status;
    if (inter <= 0 || inter % 128) return MOE_ERR_SHAPE;
    if (n_blocks > 0 && !ac) return MOE_ERR_NULL;
    WgSrc s{nullptr, nullptr, nullptr, nullptr, ac, 0, 1, inter};
    return launch_wgrad_quant<kWgH>(s, blocks, n_blocks, inter, ht, ht_scales, stream);
}

extern "C" MOE_API int moe_wgrad_quant_dac(const float* dh, const float* ac, int inter,
                                           const int32_t* blocks, int n_blocks, uint8_t* dact,
                                           float* dact_scales, int* dev_status, void* stream) {
    (void)dev_status;
    if (inter <= 0 || inter % 128) return MOE_ERR_SHAPE;
    if (n_blocks > 0 && (!dh || !ac)) return MOE_ERR_NULL;
    WgSrc s{nullptr, nullptr, nullptr, dh, ac, 0, 1, inter};
    return launch_wgrad_quant<kWgDac>(s, blocks, n_blocks, 2 * inter, dact, dact_scales, stream);
}
