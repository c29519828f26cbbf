// Single-GPU dispatch and combine of the MoE block ("DeepSeek-V3 Technical
// Report" notes page, section "DualPipe": all-to-all dispatch / combine of
// each chunk; section "FP8 mixed precision training": FP8 activations are
// what is dispatched) and the bias update of section "DeepSeekMoE and
// auxiliary-loss-free load balancing".
//
// moe_permute builds an expert-contiguous copy of the FP8 token rows:
//   1. chunk_hist: per chunk of kChunk tokens, how many of its pairs go to
//      each expert (scratch [n_chunks, N_r]);
//   2. chunk_scan: per expert, the exclusive scan of those counts over
//      chunks plus the expert's base offset -> first row of each
//      (chunk, expert); block 0 also writes expert_offsets;
//   3. chunk_rank: per chunk, one warp walks its tokens in order and hands
//      out rows (tokens stay in ascending order inside every expert);
//   4. copy_rows: one warp per token reads its FP8 row once (16-byte loads)
//      and writes it K+1 times, scales transposed to the kb-major layout.
#include <mutex>

#include <algorithm>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kChunk = 64;

__global__ void __launch_bounds__(256) chunk_hist_kernel(const int32_t* __restrict__ topk_idx,
                                                         int T, int K, int n_routed,
                                                         int32_t* __restrict__ chunk_counts,
                                                         int* dev_status) {
    extern __shared__ int hist_smem[];
    for (int i = threadIdx.x; i < n_routed; i += blockDim.x) hist_smem[i] = 0;
    __syncthreads();
    const int t0 = blockIdx.x * kChunk;
    const int t1 = min(T, t0 + kChunk);
    for (int p = t0 * K + threadIdx.x; p < t1 * K; p += blockDim.x) {
        const int e = topk_idx[p];
        if (e < 0 || e >= n_routed) set_status(dev_status, MOE_DEV_BAD_INPUT);
        else atomicAdd(&hist_smem[e], 1);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < n_routed; i += blockDim.x)
        chunk_counts[int64_t(blockIdx.x) * n_routed + i] = hist_smem[i];
}

// One block (256 threads) per expert e.  Exclusive scan over chunks of
// chunk_counts[., e], plus off[e] = sum of counts of experts < e.
__global__ void __launch_bounds__(256) chunk_scan_kernel(const int32_t* __restrict__ counts,
                                                         int T, int K, int n_routed, int n_chunks,
                                                         int32_t* __restrict__ chunk_counts,
                                                         int32_t* __restrict__ expert_offsets) {
    __shared__ int warp_sums[8];
    __shared__ int base_s;
    const int e = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // base offset of expert e
    int part = 0;
    for (int i = tid; i < e; i += 256) part += counts[i];
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (lane == 0) warp_sums[warp] = part;
    __syncthreads();
    if (tid == 0) {
        int b = 0;
        for (int w = 0; w < 8; ++w) b += warp_sums[w];
        base_s = b;
    }
    __syncthreads();
    int running = base_s;
    // scan over chunks, 256 at a time
    for (int c0 = 0; c0 < n_chunks; c0 += 256) {
        const int c = c0 + tid;
        const int v = c < n_chunks ? chunk_counts[int64_t(c) * n_routed + e] : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += n;
        }
        __syncthreads();
        if (lane == 31) warp_sums[warp] = incl;
        __syncthreads();
        int before = 0, total = 0;
        for (int w = 0; w < 8; ++w) {
            const int ws = warp_sums[w];
            if (w < warp) before += ws;
            total += ws;
        }
        if (c < n_chunks) chunk_counts[int64_t(c) * n_routed + e] = running + before + incl - v;
        running += total;
    }
    if (e == 0) {
        // expert_offsets: serial prefix by thread 0 (N_r <= 1024 values)
        __syncthreads();
        if (tid == 0) {
            int acc = 0;
            for (int i = 0; i < n_routed; ++i) {
                expert_offsets[i] = acc;
                acc += counts[i];
            }
            expert_offsets[n_routed] = acc;
            expert_offsets[n_routed + 1] = acc + T;
        }
    }
}

// One warp per chunk: tokens in ascending order; lane k < K takes slot k of
// the token (the K experts of a token are distinct, so no two lanes touch
// the same cursor in one step).  The chunk's expert ids and the experts' row
// limits are staged in shared memory first, so the serial walk touches no
// global memory except the row_of_pair stores.
__global__ void __launch_bounds__(32) chunk_rank_kernel(const int32_t* __restrict__ topk_idx,
                                                        int T, int K, int n_routed,
                                                        const int32_t* __restrict__ chunk_base,
                                                        const int32_t* __restrict__ offsets,
                                                        int32_t* __restrict__ row_of_pair,
                                                        int* dev_status) {
    extern __shared__ int rank_smem[];
    int* cursor = rank_smem;              // [n_routed]
    int* limit = rank_smem + n_routed;    // [n_routed]
    int* ids = rank_smem + 2 * n_routed;  // [kChunk * K]
    const int lane = threadIdx.x;
    const int c = blockIdx.x;
    const int t0 = c * kChunk, t1 = min(T, t0 + kChunk);
    for (int i = lane; i < n_routed; i += 32) {
        cursor[i] = chunk_base[int64_t(c) * n_routed + i];
        limit[i] = offsets[i + 1];
    }
    for (int p = lane; p < (t1 - t0) * K; p += 32) ids[p] = topk_idx[int64_t(t0) * K + p];
    __syncwarp();
    bool bad = false;
    for (int t = t0; t < t1; ++t) {
        if (lane < K) {
            const int e = ids[(t - t0) * K + lane];
            int row = -1;
            if (e >= 0 && e < n_routed) {
                row = cursor[e];
                cursor[e] = row + 1;
                // expert_counts inconsistent with topk_idx: no row to give
                if (row >= limit[e]) row = -1;
            }
            bad |= row < 0;
            row_of_pair[int64_t(t) * K + lane] = row;
        }
        __syncwarp();
    }
    if (bad) set_status(dev_status, MOE_DEV_BAD_INPUT);
}

// One warp per token; the row is read once, 4 KB at a time (8 x 16 bytes
// per lane), and each piece is written K+1 times.
constexpr int kPiece = 8;

__global__ void __launch_bounds__(256) copy_rows_kernel(
    const uint4* __restrict__ xq, const float* __restrict__ xs, int T, int d, int K,
    const int32_t* __restrict__ row_of_pair, int64_t rows_total, uint4* __restrict__ xq_perm,
    float* __restrict__ xs_perm) {
    const int lane = threadIdx.x & 31;
    const int nvec = d / 16, nkb = d / 128;
    const int warps_total = gridDim.x * (blockDim.x / 32);
    for (int t = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); t < T; t += warps_total) {
        int my_row = 0;
        if (lane < K) my_row = row_of_pair[int64_t(t) * K + lane];
        const int shared_row = T * K + t;
        const uint4* src = xq + int64_t(t) * nvec;
        for (int c0 = 0; c0 < nvec; c0 += 32 * kPiece) {
            uint4 v[kPiece];
#pragma unroll
            for (int j = 0; j < kPiece; ++j) {
                const int c = c0 + lane + 32 * j;
                if (c < nvec) v[j] = __ldcs(src + c);
            }
            for (int k = 0; k <= K; ++k) {
                const int row = (k < K) ? __shfl_sync(0xffffffffu, my_row, k) : shared_row;
                if (row < 0) continue;
                uint4* dst = xq_perm + int64_t(row) * nvec;
#pragma unroll
                for (int j = 0; j < kPiece; ++j) {
                    const int c = c0 + lane + 32 * j;
                    if (c < nvec) dst[c] = v[j];
                }
            }
        }
        for (int k = 0; k <= K; ++k) {
            const int row = (k < K) ? __shfl_sync(0xffffffffu, my_row, k) : shared_row;
            if (row < 0) continue;
            for (int kb = lane; kb < nkb; kb += 32)
                xs_perm[int64_t(kb) * rows_total + row] = xs[int64_t(t) * nkb + kb];
        }
    }
}

// moe_quant_permute's copy: a work unit is one piece of 2P tiles (P = 7 or
// 8, up to 2,048 values) of a token's bf16 row (a warp, 16-byte loads, P per
// lane in flight), so a small batch still spreads over every SM.  The warp quantises each 1x128
// tile of the piece exactly as fp8_quant_act_1x128 does (a half-warp owns
// one tile: amax by shuffles, scale rule of quant.cu, RN products, satfinite
// E4M3) and writes the codes and the scale K+1 times (routed rows and the
// shared row).
// P: 16-byte vectors per lane per piece (a piece is 2P tiles of 128 values);
// the launch picks P so that the pieces tile a row exactly when it can.
// POW2: power-of-two scales, written as UE8M0 bytes to xsf_perm instead of
// fp32 scales to xs_perm (the block-scaled GEMM's operand layout).
template <int P, bool POW2>
__global__ void __launch_bounds__(256) quant_copy_rows_kernel(
    const uint4* __restrict__ x, int T, int d, int K, const int32_t* __restrict__ row_of_pair,
    int64_t rows_total, uint2* __restrict__ xq_perm, float* __restrict__ xs_perm,
    uint8_t* __restrict__ xsf_perm) {
    constexpr int kPiece = P;
    const int lane = threadIdx.x & 31;
    const int nvec = d / 8, nkb = d / 128;  // 8 bf16 in, 8 codes out per vector
    const int pieces = (nvec + 32 * kPiece - 1) / (32 * kPiece);
    const int64_t units = int64_t(T) * pieces;
    const int64_t warps_total = int64_t(gridDim.x) * (blockDim.x / 32);
    for (int64_t un = int64_t(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5); un < units;
         un += warps_total) {
        const int t = int(un / pieces);
        int my_row = 0;
        if (lane < K) my_row = row_of_pair[int64_t(t) * K + lane];
        const int shared_row = T * K + t;
        const uint4* src = x + int64_t(t) * nvec;
        {
            const int c0 = int(un - int64_t(t) * pieces) * (32 * kPiece);
            uint4 v[kPiece];
#pragma unroll
            for (int j = 0; j < kPiece; ++j) {
                const int c = c0 + lane + 32 * j;
                v[j] = c < nvec ? __ldcs(src + c) : make_uint4(0u, 0u, 0u, 0u);
            }
            uint2 code[kPiece];
            float tile_scale = 1.0f;  // lane L < 2P: scale of tile c0/16 + L
#pragma unroll
            for (int j = 0; j < kPiece; ++j) {
                const uint4 w = v[j];
                const float f[8] = {bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y),
                                    bf16_lo(w.z), bf16_hi(w.z), bf16_lo(w.w), bf16_hi(w.w)};
                float amax = 0.0f;
#pragma unroll
                for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
#pragma unroll
                for (int o = 8; o >= 1; o >>= 1)
                    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                float scale, inv;
                if (POW2) {
                    const int e = pow2_exponent(amax);
                    inv = pow2_inverse(e);
                    scale = __int_as_float(e + 127);  // carries the byte, not a value
                } else {
                    scale_from_amax(amax, scale, inv);
                }
                const uint32_t c0_ = e4m3x2(__fmul_rn(f[0], inv), __fmul_rn(f[1], inv));
                const uint32_t c1_ = e4m3x2(__fmul_rn(f[2], inv), __fmul_rn(f[3], inv));
                const uint32_t c2_ = e4m3x2(__fmul_rn(f[4], inv), __fmul_rn(f[5], inv));
                const uint32_t c3_ = e4m3x2(__fmul_rn(f[6], inv), __fmul_rn(f[7], inv));
                code[j] = make_uint2(c0_ | (c1_ << 16), c2_ | (c3_ << 16));
                // piece j holds tiles 2j (lanes 0-15) and 2j+1 (lanes 16-31)
                const float sj = __shfl_sync(0xffffffffu, scale, (lane & 1) * 16);
                if ((lane >> 1) == j) tile_scale = sj;
            }
            const int tile = c0 / 16 + lane;
            for (int k = 0; k <= K; ++k) {
                const int row = (k < K) ? __shfl_sync(0xffffffffu, my_row, k) : shared_row;
                if (row < 0) continue;
                uint2* dst = xq_perm + int64_t(row) * nvec;
#pragma unroll
                for (int j = 0; j < kPiece; ++j) {
                    const int c = c0 + lane + 32 * j;
                    if (c < nvec) dst[c] = code[j];
                }
                if (lane < 2 * kPiece && tile < nkb) {
                    if (POW2) xsf_perm[int64_t(tile) * rows_total + row] =
                        uint8_t(__float_as_int(tile_scale));
                    else xs_perm[int64_t(tile) * rows_total + row] = tile_scale;
                }
            }
        }
    }
}

// y[t] = o[shared row] + sum_k g[t,k] * o[row_of_pair[t,k]] (fp32, slot
// order), rounded once to bf16.  A work unit is one token's 64-float4 slice
// of the row (a warp, two float4 per lane), so a small batch still spreads
// over every SM; the rows of four slots are loaded before their FMAs, which
// keeps eight 16-byte loads in flight per lane.
constexpr int kCombineU = 2;      // float4 per lane per unit
constexpr int kCombineSlots = 4;  // slots whose loads are issued together

__global__ void __launch_bounds__(256) combine_kernel(const float4* __restrict__ o, int T, int d,
                                                      int K, const int32_t* __restrict__ rop,
                                                      const float* __restrict__ gate,
                                                      uint2* __restrict__ y, int* dev_status) {
    const int lane = threadIdx.x & 31;
    const int nv = d / 4;  // float4 per row, a multiple of 32
    const int chunks = (nv + 32 * kCombineU - 1) / (32 * kCombineU);
    const int64_t units = int64_t(T) * chunks;
    const int64_t warps_total = int64_t(gridDim.x) * (blockDim.x / 32);
    for (int64_t u = int64_t(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5); u < units;
         u += warps_total) {
        const int t = int(u / chunks);
        const int c0 = int(u - int64_t(t) * chunks) * (32 * kCombineU) + lane;
        int my_row = 0;
        float my_g = 0.0f;
        if (lane < K) {
            my_row = rop[int64_t(t) * K + lane];
            my_g = gate[int64_t(t) * K + lane];
            if (my_row < 0 || my_row >= T * K) {  // skipped: contributes nothing
                set_status(dev_status, MOE_DEV_BAD_INPUT);
                my_row = T * K + t;
                my_g = 0.0f;
            }
        }
        const int64_t shared_row = int64_t(T) * K + t;
        bool on[kCombineU];
        float4 acc[kCombineU];
#pragma unroll
        for (int j = 0; j < kCombineU; ++j) {
            on[j] = c0 + 32 * j < nv;
            acc[j] = on[j] ? __ldcs(o + shared_row * nv + c0 + 32 * j) : make_float4(0, 0, 0, 0);
        }
        for (int k0 = 0; k0 < K; k0 += kCombineSlots) {
            float4 v[kCombineSlots][kCombineU];
            float g[kCombineSlots];
#pragma unroll
            for (int s = 0; s < kCombineSlots; ++s) {
                const int k = min(k0 + s, K - 1);
                const int row = __shfl_sync(0xffffffffu, my_row, k);
                g[s] = __shfl_sync(0xffffffffu, my_g, k);
#pragma unroll
                for (int j = 0; j < kCombineU; ++j)
                    v[s][j] = (on[j] && k0 + s < K) ? __ldcs(o + int64_t(row) * nv + c0 + 32 * j)
                                                    : make_float4(0, 0, 0, 0);
            }
#pragma unroll
            for (int s = 0; s < kCombineSlots; ++s) {
                if (k0 + s >= K) break;
#pragma unroll
                for (int j = 0; j < kCombineU; ++j) {
                    acc[j].x = __fmaf_rn(g[s], v[s][j].x, acc[j].x);
                    acc[j].y = __fmaf_rn(g[s], v[s][j].y, acc[j].y);
                    acc[j].z = __fmaf_rn(g[s], v[s][j].z, acc[j].z);
                    acc[j].w = __fmaf_rn(g[s], v[s][j].w, acc[j].w);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < kCombineU; ++j) {
            if (!on[j]) continue;
            __nv_bfloat162 lo = __floats2bfloat162_rn(acc[j].x, acc[j].y);
            __nv_bfloat162 hi = __floats2bfloat162_rn(acc[j].z, acc[j].w);
            y[int64_t(t) * nv + c0 + 32 * j] =
                make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
        }
    }
}

__global__ void update_bias_kernel(const int32_t* __restrict__ counts, int n_routed,
                                   int64_t total, float gamma, float* __restrict__ bias) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n_routed) return;
    const int64_t c = int64_t(counts[i]) * n_routed;
    if (c > total) bias[i] = __fsub_rn(bias[i], gamma);
    else if (c < total) bias[i] = __fadd_rn(bias[i], gamma);
}

int n_chunks_of(int T) { return (T + kChunk - 1) / kChunk; }

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" MOE_API size_t moe_permute_workspace_size(const MoeShape* shape) {
    if (validate_shape(shape) != MOE_OK) return 0;
    return align_up(size_t(n_chunks_of(shape->T)) * shape->n_routed * sizeof(int32_t) + 256, 256);
}

namespace moe {
namespace {

// Steps 1-3 of the permutation (offsets and row_of_pair); returns the
// status.  T > 0 is checked by the caller.
int build_rows(const MoeShape* shape, const int32_t* topk_idx, const int32_t* expert_counts,
               int32_t* expert_offsets, int32_t* row_of_pair, int32_t* chunk_counts,
               int* dev_status, cudaStream_t st) {
    const int T = shape->T, K = shape->topk, N = shape->n_routed;
    const int n_chunks = n_chunks_of(T);
    int rc;
    if (T > 0) {
        chunk_hist_kernel<<<n_chunks, 256, sizeof(int) * N, st>>>(topk_idx, T, K, N,
                                                                   chunk_counts, dev_status);
        if ((rc = check_launch()) != MOE_OK) return rc;
    }
    chunk_scan_kernel<<<N, 256, 0, st>>>(expert_counts, T, K, N, n_chunks, chunk_counts,
                                         expert_offsets);
    if ((rc = check_launch()) != MOE_OK) return rc;
    if (T == 0) return MOE_OK;
    const size_t rank_smem = sizeof(int) * (2 * size_t(N) + size_t(kChunk) * K);
    chunk_rank_kernel<<<n_chunks, 32, rank_smem, st>>>(topk_idx, T, K, N, chunk_counts,
                                                       expert_offsets, row_of_pair, dev_status);
    return check_launch();
}

// quantise + copy pass of moe_quant_permute (xsf_perm != NULL: power-of-two
// scales as UE8M0 bytes).  Pieces of 2P tiles: P = 7 cuts a 56-tile row
// (d = 7168) into four full pieces; otherwise 8, the last piece of a row
// possibly ragged.
int launch_quant_copy(const uint16_t* x, int T, int d, int K, const int32_t* row_of_pair,
                      uint8_t* xq_perm, float* xs_perm, uint8_t* xsf_perm, cudaStream_t st) {
    const int nkb = d / 128;
    const int P = (nkb % 14 == 0 && nkb % 16 != 0) ? 7 : 8;
    const int64_t pieces = (d / 8 + 32 * P - 1) / (32 * P);
    const int64_t units = int64_t(T) * pieces;  // one warp each, 8 per block
    const int qblocks = int(std::min<int64_t>((units + 7) / 8, int64_t(sm_count()) * 8));
    const uint4* xv = reinterpret_cast<const uint4*>(x);
    uint2* qv = reinterpret_cast<uint2*>(xq_perm);
    const int64_t rows = int64_t(T) * K + T;
    if (P == 7 && xsf_perm)
        quant_copy_rows_kernel<7, true><<<qblocks, 256, 0, st>>>(xv, T, d, K, row_of_pair, rows,
                                                                 qv, xs_perm, xsf_perm);
    else if (P == 7)
        quant_copy_rows_kernel<7, false><<<qblocks, 256, 0, st>>>(xv, T, d, K, row_of_pair, rows,
                                                                  qv, xs_perm, xsf_perm);
    else if (xsf_perm)
        quant_copy_rows_kernel<8, true><<<qblocks, 256, 0, st>>>(xv, T, d, K, row_of_pair, rows,
                                                                 qv, xs_perm, xsf_perm);
    else
        quant_copy_rows_kernel<8, false><<<qblocks, 256, 0, st>>>(xv, T, d, K, row_of_pair, rows,
                                                                  qv, xs_perm, xsf_perm);
    return check_launch();
}

int copy_grid(int T) {
    int blocks = (T + 7) / 8;
    const int cap = sm_count() * 8;
    return blocks > cap ? cap : blocks;
}

}  // namespace
}  // namespace moe

extern "C" MOE_API int moe_permute(const MoeShape* shape, const int32_t* topk_idx,
                                   const int32_t* expert_counts, const uint8_t* xq,
                                   const float* xs, uint8_t* xq_perm, float* xs_perm,
                                   int32_t* expert_offsets, int32_t* row_of_pair, void* ws,
                                   size_t ws_bytes, int* dev_status, void* stream) {
    int rc = validate_shape(shape);
    if (rc != MOE_OK) return rc;
    const int T = shape->T, d = shape->d, K = shape->topk;
    if (!expert_counts || !expert_offsets) return MOE_ERR_NULL;
    if (T > 0) {
        if (!topk_idx || !xq || !xs || !xq_perm || !xs_perm || !row_of_pair) return MOE_ERR_NULL;
        if (!aligned16(xq) || !aligned16(xq_perm)) return MOE_ERR_ALIGN;
        if (!ws || ws_bytes < moe_permute_workspace_size(shape)) return MOE_ERR_WORKSPACE;
    }
    cudaStream_t st = as_stream(stream);
    rc = build_rows(shape, topk_idx, expert_counts, expert_offsets, row_of_pair,
                    static_cast<int32_t*>(ws), dev_status, st);
    if (rc != MOE_OK || T == 0) return rc;
    copy_rows_kernel<<<copy_grid(T), 256, 0, st>>>(
        reinterpret_cast<const uint4*>(xq), xs, T, d, K, row_of_pair, int64_t(T) * K + T,
        reinterpret_cast<uint4*>(xq_perm), xs_perm);
    return check_launch();
}

extern "C" MOE_API int moe_quant_permute(const MoeShape* shape, const uint16_t* x,
                                         const int32_t* topk_idx, const int32_t* expert_counts,
                                         uint8_t* xq_perm, float* xs_perm,
                                         int32_t* expert_offsets, int32_t* row_of_pair, void* ws,
                                         size_t ws_bytes, int* dev_status, void* stream) {
    int rc = validate_shape(shape);
    if (rc != MOE_OK) return rc;
    const int T = shape->T, d = shape->d, K = shape->topk;
    if (!expert_counts || !expert_offsets) return MOE_ERR_NULL;
    if (T > 0) {
        if (!topk_idx || !x || !xq_perm || !xs_perm || !row_of_pair) return MOE_ERR_NULL;
        if (!aligned16(x) || !aligned16(xq_perm) || (reinterpret_cast<uintptr_t>(xs_perm) & 3))
            return MOE_ERR_ALIGN;
        if (!ws || ws_bytes < moe_permute_workspace_size(shape)) return MOE_ERR_WORKSPACE;
    }
    cudaStream_t st = as_stream(stream);
    rc = build_rows(shape, topk_idx, expert_counts, expert_offsets, row_of_pair,
                    static_cast<int32_t*>(ws), dev_status, st);
    if (rc != MOE_OK || T == 0) return rc;
    return launch_quant_copy(x, T, d, K, row_of_pair, xq_perm, xs_perm, nullptr, st);
}

extern "C" MOE_API int moe_quant_permute_ue8m0(const MoeShape* shape, const uint16_t* x,
                                               const int32_t* topk_idx,
                                               const int32_t* expert_counts, uint8_t* xq_perm,
                                               uint8_t* xsf_perm, int32_t* expert_offsets,
                                               int32_t* row_of_pair, void* ws, size_t ws_bytes,
                                               int* dev_status, void* stream) {
    int rc = validate_shape(shape);
    if (rc != MOE_OK) return rc;
    const int T = shape->T, d = shape->d, K = shape->topk;
    if (!expert_counts || !expert_offsets) return MOE_ERR_NULL;
    if (T > 0) {
        if (!topk_idx || !x || !xq_perm || !xsf_perm || !row_of_pair) return MOE_ERR_NULL;
        if (!aligned16(x) || !aligned16(xq_perm)) return MOE_ERR_ALIGN;
        if (!ws || ws_bytes < moe_permute_workspace_size(shape)) return MOE_ERR_WORKSPACE;
    }
    cudaStream_t st = as_stream(stream);
    rc = build_rows(shape, topk_idx, expert_counts, expert_offsets, row_of_pair,
                    static_cast<int32_t*>(ws), dev_status, st);
    if (rc != MOE_OK || T == 0) return rc;
    return launch_quant_copy(x, T, d, K, row_of_pair, xq_perm, nullptr, xsf_perm, st);
}

extern "C" MOE_API int moe_combine(const MoeShape* shape, const float* expert_out,
                                   const int32_t* expert_offsets, const int32_t* row_of_pair,
                                   const float* topk_gate, uint16_t* y, int* dev_status,
                                   void* stream) {
    (void)expert_offsets;
    int rc = validate_shape(shape);
    if (rc != MOE_OK) return rc;
    const int T = shape->T;
    if (T == 0) return MOE_OK;
    if (!expert_out || !row_of_pair || !topk_gate || !y) return MOE_ERR_NULL;
    if (!aligned16(expert_out) || (reinterpret_cast<uintptr_t>(y) & 7)) return MOE_ERR_ALIGN;
    const int64_t chunks = (shape->d / 4 + 32 * kCombineU - 1) / (32 * kCombineU);
    const int64_t units = int64_t(T) * chunks;  // one warp each, 8 per block
    const int64_t cap = int64_t(sm_count()) * 8;
    const int blocks = int(std::min<int64_t>((units + 7) / 8, cap));
    combine_kernel<<<blocks, 256, 0, as_stream(stream)>>>(
        reinterpret_cast<const float4*>(expert_out), T, shape->d, shape->topk, row_of_pair,
        topk_gate, reinterpret_cast<uint2*>(y), dev_status);
    return check_launch();
}

extern "C" MOE_API int moe_update_bias(const MoeShape* shape, const int32_t* expert_counts,
                                       float* bias, int* dev_status, void* stream) {
    (void)dev_status;
    int rc = validate_shape(shape);
    if (rc != MOE_OK) return rc;
    if (!expert_counts || !bias) return MOE_ERR_NULL;
    const int N = shape->n_routed;
    update_bias_kernel<<<(N + 255) / 256, 256, 0, as_stream(stream)>>>(
        expert_counts, N, int64_t(shape->T) * shape->topk, shape->gamma, bias);
    return check_launch();
}

// ------------------------------------------------------------------------
// moe_permute_static_ws: moe_permute without a caller workspace.
//
// Some callers cannot call cudaMalloc once they are running: a serving loop
// whose device-memory budget is fixed when it starts, or a host framework
// that owns all device memory through its own pool and forbids allocations
// behind its back (cudaMalloc may also synchronise the whole device, which
// latency-bound loops avoid).  This entry point lets them run the
// permutation without sizing or passing a workspace: the per-chunk counts
// live in the array below, which every GPU that loads the library keeps
// until the process exits.
namespace moe {
namespace {

constexpr int64_t kStaticChunkEntries = 262144;  // int32 entries = 1 MiB
// + 64 entries: moe_permute asks for 256 bytes of headroom on top of the counts
__device__ __align__(256) int32_t g_permute_scratch[kStaticChunkEntries + 64];

// Unique id of the calling thread's current CUDA context (cuCtxGetId through
// the runtime's driver entry points), or 0 when there is none or the driver
// cannot tell.
unsigned long long current_context_id() {
    typedef int (*GetCurrentFn)(void**);
    typedef int (*GetIdFn)(void*, unsigned long long*);
    static GetCurrentFn get_current = nullptr;
    static GetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrentFn>(f);
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetIdFn>(f);
    });
    void* ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != 0 || !ctx || get_id(ctx, &id) != 0)
        return 0;
    return id;
}

// Device address of g_permute_scratch in the current device's context.  In
// host code the symbol only names a host-side stand-in, never a device
// address.  The address is looked up once per device and context: a device
// reset ends the context it belongs to, and the next call, seeing a new
// context id, looks it up again.
int32_t* static_scratch_ptr() {
    static std::mutex mu;
    static int32_t* ptrs[64] = {nullptr};
    static unsigned long long ctx_ids[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    const unsigned long long id = current_context_id();
    if (!ptrs[dev] || id == 0 || id != ctx_ids[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess) return nullptr;
        ptrs[dev] = static_cast<int32_t*>(p);
        ctx_ids[dev] = current_context_id();  // the lookup made the context current
    }
    return ptrs[dev];
}

}  // namespace
}  // namespace moe

extern "C" MOE_API int moe_permute_static_ws(const MoeShape* shape, const int32_t* topk_idx,
                                             const int32_t* expert_counts, const uint8_t* xq,
                                             const float* xs, uint8_t* xq_perm, float* xs_perm,
                                             int32_t* expert_offsets, int32_t* row_of_pair,
                                             int* dev_status, void* stream) {
    int rc = validate_shape(shape);
    if (rc != MOE_OK) return rc;
    if (int64_t(n_chunks_of(shape->T)) * shape->n_routed > kStaticChunkEntries)
        return MOE_ERR_STATIC_LIMIT;
    int32_t* scratch = static_scratch_ptr();
    if (!scratch) return MOE_ERR_CUDA;
    // The scratch needs no clearing: chunk_hist writes every entry that the
    // later kernels of this call read.
    return moe_permute(shape, topk_idx, expert_counts, xq, xs, xq_perm, xs_perm, expert_offsets,
                       row_of_pair, scratch, sizeof(g_permute_scratch), dev_status, stream);
}
