// Expert parallelism: dispatch and combine of the MoE block across P ranks
// ("DeepSeek-V3 Technical Report" notes page, section "DualPipe": all-to-all
// dispatch and combine around the expert MLP, each token sent to at most
// M = 4 nodes; section "FP8 mixed precision training": the dispatched
// activations are FP8).  Rank q owns routed experts [q E, (q+1) E) with
// E = N_r / P; every rank runs the shared expert on its own tokens.  A token
// travels once to each rank that owns at least one of its K experts (group-
// limited routing bounds that to M ranks when the groups are the ranks), as
// one row: its FP8 codes, its 1x128 scales, and its slots on that rank.
//
// Row layout (moe_ep_row_bytes): codes uint8 [d] | scales fp32 [d/128] |
// local expert of each slot int32 [K] (-1: the slot's expert is elsewhere) |
// gate of each slot fp32 [K] | source token int32 | zero padding to 16 bytes.
//
// The exchange itself (two all-to-alls of rows and one of fp32 partial
// outputs, with the counts) is NCCL's, driven by the caller; these kernels
// build, consume and combine the buffers:
//   1. ep_plan_*: destinations of every token, rows per destination, and the
//      row of each (token, destination) in the send buffer (destination-major,
//      tokens ascending);
//   2. ep_pack_kernel: x read once in bf16, each 1x128 tile quantised (the
//      scale rule of fp8_quant_act_1x128) into every destination row;
//   3. ep_local_*: the received rows -> expert-contiguous FP8 rows of the
//      local experts (received order kept inside an expert), the operands of
//      moe_grouped_gemm_fp8;
//   4. ep_partial_combine_kernel: per received row, the gate-weighted sum of
//      its local experts' outputs (fp32, slot order), sent back;
//   5. ep_final_combine_kernel: y = shared expert output + the partial sums of
//      the token's destinations in rank order, rounded once to bf16.
#include <algorithm>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kEpChunk = 64;

struct RowLayout {
    int64_t codes, scales, slots, gates, src, bytes;
};

__host__ __device__ inline RowLayout row_layout(int d, int K) {
    RowLayout r;
    r.codes = 0;
    r.scales = d;
    r.slots = r.scales + 4 * (d / 128);
    r.gates = r.slots + 4 * K;
    r.src = r.gates + 4 * K;
    r.bytes = (r.src + 4 + 15) / 16 * 16;
    return r;
}

// ------------------------------------------------------------ 1. plan
// Destination mask of each token (bit q: one of its experts lives on rank q).
__global__ void ep_mask_kernel(const int32_t* __restrict__ topk_idx, int T, int K, int E,
                               int P, uint32_t* __restrict__ mask, int* dev_status) {
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T) return;
    uint32_t m = 0;
    for (int k = 0; k < K; ++k) {
        const int e = topk_idx[int64_t(t) * K + k];
        const int q = e >= 0 ? e / E : -1;
        if (q < 0 || q >= P) set_status(dev_status, MOE_DEV_BAD_INPUT);
        else m |= 1u << q;
    }
    mask[t] = m;
}

// One block per destination q: the rank of every token with bit q among the
// tokens before it (block-wide scan, 1024 tokens per pass); the row is
// assigned once the offsets are known (counts first, then rows).
template <bool ROWS>
__global__ void __launch_bounds__(1024) ep_scan_kernel(const uint32_t* __restrict__ mask, int T,
                                                       int P, int32_t* __restrict__ counts,
                                                       const int32_t* __restrict__ offsets,
                                                       int32_t* __restrict__ send_row) {
    __shared__ int wsum[32];
    const int q = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int running = ROWS ? offsets[q] : 0;
    for (int t0 = 0; t0 < T; t0 += 1024) {
        const int t = t0 + threadIdx.x;
        const int bit = t < T ? int((mask[t] >> q) & 1u) : 0;
        const unsigned b = __ballot_sync(0xffffffffu, bit);
        const int before_in_warp = __popc(b & ((1u << lane) - 1u));
        if (lane == 0) wsum[warp] = __popc(b);
        __syncthreads();
        int before = 0, total = 0;
        for (int w = 0; w < 32; ++w) {
            if (w < warp) before += wsum[w];
            total += wsum[w];
        }
        if (ROWS && t < T) send_row[int64_t(t) * P + q] = bit ? running + before + before_in_warp : -1;
        running += total;
        __syncthreads();
    }
    if (!ROWS && threadIdx.x == 0) counts[q] = running;
}

__global__ void ep_offsets_kernel(const int32_t* __restrict__ counts, int P,
                                  int32_t* __restrict__ offsets) {
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int q = 0; q < P; ++q) {
            offsets[q] = acc;
            acc += counts[q];
        }
        offsets[P] = acc;
    }
}

// ------------------------------------------------------------ 2. pack
// A warp per (token, piece of 2P tiles): the piece is read once in bf16,
// each 1x128 tile quantised by a half-warp, and the codes and scales written
// to every destination row of the token; the warp of piece 0 also writes the
// slots, gates and source token of each row.
template <int PC>
__global__ void __launch_bounds__(256) ep_pack_kernel(
    const uint4* __restrict__ x, int T, int d, int K, int E, int P,
    const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_gate,
    const int32_t* __restrict__ send_row, uint8_t* __restrict__ send_buf) {
    const int lane = threadIdx.x & 31;
    const RowLayout L = row_layout(d, K);
    const int nvec = d / 8, nkb = d / 128;
    const int pieces = (nvec + 32 * PC - 1) / (32 * PC);
    const int64_t units = int64_t(T) * pieces;
    const int64_t warps_total = int64_t(gridDim.x) * (blockDim.x / 32);
    for (int64_t un = int64_t(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5); un < units;
         un += warps_total) {
        const int t = int(un / pieces);
        const int piece = int(un - int64_t(t) * pieces);
        const int c0 = piece * 32 * PC;
        const uint4* src = x + int64_t(t) * nvec;
        uint4 v[PC];
#pragma unroll
        for (int j = 0; j < PC; ++j) {
            const int c = c0 + lane + 32 * j;
            v[j] = c < nvec ? __ldcs(src + c) : make_uint4(0u, 0u, 0u, 0u);
        }
        uint2 code[PC];
        float tile_scale = 1.0f;  // lane L < 2 PC: scale of tile c0/16 + L
#pragma unroll
        for (int j = 0; j < PC; ++j) {
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
            scale_from_amax(amax, scale, inv);
            const uint32_t a0 = e4m3x2(__fmul_rn(f[0], inv), __fmul_rn(f[1], inv));
            const uint32_t a1 = e4m3x2(__fmul_rn(f[2], inv), __fmul_rn(f[3], inv));
            const uint32_t a2 = e4m3x2(__fmul_rn(f[4], inv), __fmul_rn(f[5], inv));
            const uint32_t a3 = e4m3x2(__fmul_rn(f[6], inv), __fmul_rn(f[7], inv));
            code[j] = make_uint2(a0 | (a1 << 16), a2 | (a3 << 16));
            const float sj = __shfl_sync(0xffffffffu, scale, (lane & 1) * 16);
            if ((lane >> 1) == j) tile_scale = sj;
        }
        const int tile = c0 / 16 + lane;
        for (int q = 0; q < P; ++q) {
            const int row = send_row[int64_t(t) * P + q];
            if (row < 0) continue;
            uint8_t* dst = send_buf + int64_t(row) * L.bytes;
            uint2* cd = reinterpret_cast<uint2*>(dst + L.codes);
#pragma unroll
            for (int j = 0; j < PC; ++j) {
                const int c = c0 + lane + 32 * j;
                if (c < nvec) cd[c] = code[j];
            }
            if (lane < 2 * PC && tile < nkb)
                reinterpret_cast<float*>(dst + L.scales)[tile] = tile_scale;
            if (piece == 0) {
                if (lane < K) {
                    const int e = topk_idx[int64_t(t) * K + lane];
                    const bool here = e >= 0 && e / E == q;
                    reinterpret_cast<int32_t*>(dst + L.slots)[lane] = here ? e - q * E : -1;
                    reinterpret_cast<float*>(dst + L.gates)[lane] =
                        here ? topk_gate[int64_t(t) * K + lane] : 0.0f;
                }
                if (lane == 0) *reinterpret_cast<int32_t*>(dst + L.src) = t;
                for (int64_t b = L.src + 4 + lane; b < L.bytes; b += 32) dst[b] = 0;
            }
        }
    }
}

// ------------------------------------------------------------ 3. local rows
// Per chunk of received rows: how many of its slots go to each local expert;
// totals per expert accumulate atomically (integer: order-free).
__global__ void __launch_bounds__(256) ep_chunk_hist_kernel(
    const uint8_t* __restrict__ recv, int n_recv, int d, int K, int E,
    int32_t* __restrict__ chunk_counts, int32_t* __restrict__ totals, int* dev_status) {
    extern __shared__ int ep_hist[];
    const RowLayout L = row_layout(d, K);
    for (int i = threadIdx.x; i < E; i += blockDim.x) ep_hist[i] = 0;
    __syncthreads();
    const int r0 = blockIdx.x * kEpChunk, r1 = min(n_recv, r0 + kEpChunk);
    for (int p = r0 * K + threadIdx.x; p < r1 * K; p += blockDim.x) {
        const int r = p / K, k = p - r * K;
        const int e = reinterpret_cast<const int32_t*>(recv + int64_t(r) * L.bytes + L.slots)[k];
        if (e < 0) continue;  // the slot's expert is on another rank
        if (e >= E) set_status(dev_status, MOE_DEV_BAD_INPUT);
        else atomicAdd(&ep_hist[e], 1);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < E; i += blockDim.x) {
        chunk_counts[int64_t(blockIdx.x) * E + i] = ep_hist[i];
        if (ep_hist[i]) atomicAdd(&totals[i], ep_hist[i]);
    }
}

// One block per local expert: exclusive scan of its chunk counts plus the
// expert's base offset; block 0 writes the offsets [E + 1].
__global__ void __launch_bounds__(256) ep_chunk_scan_kernel(const int32_t* __restrict__ totals,
                                                            int E, int n_chunks,
                                                            int32_t* __restrict__ chunk_counts,
                                                            int32_t* __restrict__ offsets) {
    __shared__ int wsum[8];
    __shared__ int base_s;
    const int e = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int part = 0;
    for (int i = tid; i < e; i += 256) part += totals[i];
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (lane == 0) wsum[warp] = part;
    __syncthreads();
    if (tid == 0) {
        int b = 0;
        for (int w = 0; w < 8; ++w) b += wsum[w];
        base_s = b;
    }
    __syncthreads();
    int running = base_s;
    for (int c0 = 0; c0 < n_chunks; c0 += 256) {
        const int c = c0 + tid;
        const int v = c < n_chunks ? chunk_counts[int64_t(c) * E + e] : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += n;
        }
        __syncthreads();
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        int before = 0, total = 0;
        for (int w = 0; w < 8; ++w) {
            if (w < warp) before += wsum[w];
            total += wsum[w];
        }
        if (c < n_chunks) chunk_counts[int64_t(c) * E + e] = running + before + incl - v;
        running += total;
    }
    if (e == 0) {
        __syncthreads();
        if (tid == 0) {
            int acc = 0;
            for (int i = 0; i < E; ++i) {
                offsets[i] = acc;
                acc += totals[i];
            }
            offsets[E] = acc;
        }
    }
}

// One warp per chunk: received rows in order, lane k < K hands slot k its row
// (a row's experts are distinct, so no two lanes share a cursor in a step).
// Rows at or past max_rows (more local slots than the caller's buffers hold)
// are not handed out: their slots get -1 and the status reports it.
__global__ void __launch_bounds__(32) ep_chunk_rank_kernel(
    const uint8_t* __restrict__ recv, int n_recv, int d, int K, int E,
    const int32_t* __restrict__ chunk_base, const int32_t* __restrict__ offsets, int max_rows,
    int32_t* __restrict__ pair_row, int* dev_status) {
    extern __shared__ int ep_cursor[];
    int* limit = ep_cursor + E;
    const RowLayout L = row_layout(d, K);
    const int lane = threadIdx.x, c = blockIdx.x;
    const int r0 = c * kEpChunk, r1 = min(n_recv, r0 + kEpChunk);
    for (int i = lane; i < E; i += 32) {
        ep_cursor[i] = chunk_base[int64_t(c) * E + i];
        limit[i] = offsets[i + 1];
    }
    __syncwarp();
    bool bad = false;
    for (int r = r0; r < r1; ++r) {
        if (lane < K) {
            const int e = reinterpret_cast<const int32_t*>(recv + int64_t(r) * L.bytes + L.slots)[lane];
            int row = -1;
            if (e >= 0 && e < E) {
                row = ep_cursor[e];
                ep_cursor[e] = row + 1;
                if (row >= limit[e] || row >= max_rows) {
                    row = -1;
                    bad = true;
                }
            }
            pair_row[int64_t(r) * K + lane] = row;
        }
        __syncwarp();
    }
    if (bad) set_status(dev_status, MOE_DEV_BAD_INPUT);
}

// A warp per received row: its codes to each of its local rows (16-byte
// vectors), its scales to the kb-major scale array.
__global__ void __launch_bounds__(256) ep_copy_rows_kernel(
    const uint8_t* __restrict__ recv, int n_recv, int d, int K,
    const int32_t* __restrict__ pair_row, int64_t rows_total, uint4* __restrict__ xq_perm,
    float* __restrict__ xs_perm) {
    const int lane = threadIdx.x & 31;
    const RowLayout L = row_layout(d, K);
    const int nvec = d / 16, nkb = d / 128;
    const int64_t warps_total = int64_t(gridDim.x) * (blockDim.x / 32);
    for (int64_t r = int64_t(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5); r < n_recv;
         r += warps_total) {
        const uint8_t* row = recv + r * L.bytes;
        int my_row = -1;
        if (lane < K) my_row = pair_row[r * K + lane];
        const uint4* src = reinterpret_cast<const uint4*>(row + L.codes);
        const float* sc = reinterpret_cast<const float*>(row + L.scales);
        for (int k = 0; k < K; ++k) {
            const int dst_row = __shfl_sync(0xffffffffu, my_row, k);
            if (dst_row < 0) continue;
            uint4* dst = xq_perm + int64_t(dst_row) * nvec;
            for (int c = lane; c < nvec; c += 32) dst[c] = src[c];
            for (int kb = lane; kb < nkb; kb += 32) xs_perm[int64_t(kb) * rows_total + dst_row] = sc[kb];
        }
    }
}

// ------------------------------------------------------------ 4., 5. combine
// A warp per (row, 64-float4 slice): the gate-weighted sum of the row's
// local outputs in slot order (fp32), or of the shared output and the
// partial sums of the token's destinations in rank order (then bf16).
constexpr int kEpU = 2;  // float4 per lane

__global__ void __launch_bounds__(256) ep_partial_combine_kernel(
    const uint8_t* __restrict__ recv, int n_recv, int d, int K,
    const int32_t* __restrict__ pair_row, const float4* __restrict__ o,
    float4* __restrict__ back) {
    const int lane = threadIdx.x & 31;
    const RowLayout L = row_layout(d, K);
    const int nv = d / 4;
    const int chunks = (nv + 32 * kEpU - 1) / (32 * kEpU);
    const int64_t units = int64_t(n_recv) * chunks;
    const int64_t warps_total = int64_t(gridDim.x) * (blockDim.x / 32);
    for (int64_t u = int64_t(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5); u < units;
         u += warps_total) {
        const int64_t r = u / chunks;
        const int c0 = int(u - r * chunks) * (32 * kEpU) + lane;
        int my_row = -1;
        float my_g = 0.0f;
        if (lane < K) {
            my_row = pair_row[r * K + lane];
            my_g = reinterpret_cast<const float*>(recv + r * L.bytes + L.gates)[lane];
        }
        float4 acc[kEpU];
#pragma unroll
        for (int j = 0; j < kEpU; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int k = 0; k < K; ++k) {
            const int row = __shfl_sync(0xffffffffu, my_row, k);
            const float g = __shfl_sync(0xffffffffu, my_g, k);
            if (row < 0) continue;
#pragma unroll
            for (int j = 0; j < kEpU; ++j) {
                const int c = c0 + 32 * j;
                if (c >= nv) continue;
                const float4 v = __ldcs(o + int64_t(row) * nv + c);
                acc[j].x = __fmaf_rn(g, v.x, acc[j].x);
                acc[j].y = __fmaf_rn(g, v.y, acc[j].y);
                acc[j].z = __fmaf_rn(g, v.z, acc[j].z);
                acc[j].w = __fmaf_rn(g, v.w, acc[j].w);
            }
        }
#pragma unroll
        for (int j = 0; j < kEpU; ++j) {
            const int c = c0 + 32 * j;
            if (c < nv) back[r * nv + c] = acc[j];
        }
    }
}

__global__ void __launch_bounds__(256) ep_final_combine_kernel(
    const float4* __restrict__ o_shared, const float4* __restrict__ back_recv, int T, int d,
    int P, const int32_t* __restrict__ send_row, uint2* __restrict__ y) {
    const int lane = threadIdx.x & 31;
    const int nv = d / 4;
    const int chunks = (nv + 32 * kEpU - 1) / (32 * kEpU);
    const int64_t units = int64_t(T) * chunks;
    const int64_t warps_total = int64_t(gridDim.x) * (blockDim.x / 32);
    for (int64_t u = int64_t(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5); u < units;
         u += warps_total) {
        const int64_t t = u / chunks;
        const int c0 = int(u - t * chunks) * (32 * kEpU) + lane;
        float4 acc[kEpU];
#pragma unroll
        for (int j = 0; j < kEpU; ++j) {
            const int c = c0 + 32 * j;
            acc[j] = c < nv ? __ldcs(o_shared + t * nv + c) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        for (int q = 0; q < P; ++q) {
            const int row = send_row[t * P + q];
            if (row < 0) continue;
#pragma unroll
            for (int j = 0; j < kEpU; ++j) {
                const int c = c0 + 32 * j;
                if (c >= nv) continue;
                const float4 v = __ldcs(back_recv + int64_t(row) * nv + c);
                acc[j].x = __fadd_rn(acc[j].x, v.x);
                acc[j].y = __fadd_rn(acc[j].y, v.y);
                acc[j].z = __fadd_rn(acc[j].z, v.z);
                acc[j].w = __fadd_rn(acc[j].w, v.w);
            }
        }
#pragma unroll
        for (int j = 0; j < kEpU; ++j) {
            const int c = c0 + 32 * j;
            if (c >= nv) continue;
            __nv_bfloat162 lo = __floats2bfloat162_rn(acc[j].x, acc[j].y);
            __nv_bfloat162 hi = __floats2bfloat162_rn(acc[j].z, acc[j].w);
            y[t * nv + c] =
                make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
        }
    }
}

int ep_check(const MoeShape* s, int P) {
    int rc = validate_shape(s);
    if (rc != MOE_OK) return rc;
    if (P < 1 || P > 32 || s->n_routed % P) return MOE_ERR_ARG;
    return MOE_OK;
}

int warp_grid(int64_t units) {
    const int64_t cap = int64_t(sm_count()) * 8;
    return int(std::max<int64_t>(1, std::min<int64_t>((units + 7) / 8, cap)));
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" MOE_API size_t moe_ep_row_bytes(const MoeShape* shape) {
    if (validate_shape(shape) != MOE_OK) return 0;
    return size_t(row_layout(shape->d, shape->topk).bytes);
}

extern "C" MOE_API size_t moe_ep_workspace_size(const MoeShape* shape, int n_ranks,
                                                int max_recv_rows) {
    if (ep_check(shape, n_ranks) != MOE_OK || max_recv_rows < 0) return 0;
    const int E = shape->n_routed / n_ranks;
    const size_t mask = align_up(sizeof(uint32_t) * std::max(shape->T, 1), 256);
    const size_t chunks = (size_t(max_recv_rows) + kEpChunk - 1) / kEpChunk;
    return mask + align_up(sizeof(int32_t) * (chunks * E + E + 64), 256);
}

extern "C" MOE_API int moe_ep_dispatch_plan(const MoeShape* shape, int n_ranks,
                                            const int32_t* topk_idx, int32_t* send_counts,
                                            int32_t* send_offsets, int32_t* send_row, void* ws,
                                            size_t ws_bytes, int* dev_status, void* stream) {
    int rc = ep_check(shape, n_ranks);
    if (rc != MOE_OK) return rc;
    const int T = shape->T, K = shape->topk, P = n_ranks, E = shape->n_routed / P;
    if (!send_counts || !send_offsets || (T > 0 && (!topk_idx || !send_row)))
        return MOE_ERR_NULL;
    if (!ws || ws_bytes < moe_ep_workspace_size(shape, P, 0)) return MOE_ERR_WORKSPACE;
    cudaStream_t st = as_stream(stream);
    uint32_t* mask = static_cast<uint32_t*>(ws);
    if (T > 0) {
        ep_mask_kernel<<<(T + 255) / 256, 256, 0, st>>>(topk_idx, T, K, E, P, mask, dev_status);
        if ((rc = check_launch()) != MOE_OK) return rc;
    }
    ep_scan_kernel<false><<<P, 1024, 0, st>>>(mask, T, P, send_counts, nullptr, nullptr);
    if ((rc = check_launch()) != MOE_OK) return rc;
    ep_offsets_kernel<<<1, 32, 0, st>>>(send_counts, P, send_offsets);
    if ((rc = check_launch()) != MOE_OK) return rc;
    if (T == 0) return MOE_OK;
    ep_scan_kernel<true><<<P, 1024, 0, st>>>(mask, T, P, nullptr, send_offsets, send_row);
    return check_launch();
}

extern "C" MOE_API int moe_ep_pack(const MoeShape* shape, int n_ranks, const uint16_t* x,
                                   const int32_t* topk_idx, const float* topk_gate,
                                   const int32_t* send_row, uint8_t* send_buf, int* dev_status,
                                   void* stream) {
    (void)dev_status;
    int rc = ep_check(shape, n_ranks);
    if (rc != MOE_OK) return rc;
    const int T = shape->T, d = shape->d, K = shape->topk, P = n_ranks;
    if (T == 0) return MOE_OK;
    if (!x || !topk_idx || !topk_gate || !send_row || !send_buf) return MOE_ERR_NULL;
    if (!aligned16(x) || !aligned16(send_buf)) return MOE_ERR_ALIGN;
    const int nkb = d / 128;
    const int PC = (nkb % 14 == 0 && nkb % 16 != 0) ? 7 : 8;
    const int64_t pieces = (d / 8 + 32 * PC - 1) / (32 * PC);
    const int grid = warp_grid(int64_t(T) * pieces);
    const uint4* xv = reinterpret_cast<const uint4*>(x);
    if (PC == 7)
        ep_pack_kernel<7><<<grid, 256, 0, as_stream(stream)>>>(
            xv, T, d, K, shape->n_routed / P, P, topk_idx, topk_gate, send_row, send_buf);
    else
        ep_pack_kernel<8><<<grid, 256, 0, as_stream(stream)>>>(
            xv, T, d, K, shape->n_routed / P, P, topk_idx, topk_gate, send_row, send_buf);
    return check_launch();
}

extern "C" MOE_API int moe_ep_local_permute(const MoeShape* shape, int n_ranks,
                                            const uint8_t* recv_buf, int n_recv,
                                            uint8_t* xq_perm, float* xs_perm, int max_rows,
                                            int32_t* local_offsets, int32_t* pair_row, void* ws,
                                            size_t ws_bytes, int* dev_status, void* stream) {
    int rc = ep_check(shape, n_ranks);
    if (rc != MOE_OK) return rc;
    const int d = shape->d, K = shape->topk, E = shape->n_routed / n_ranks;
    if (n_recv < 0 || max_rows < 0) return MOE_ERR_SHAPE;
    if (!local_offsets) return MOE_ERR_NULL;
    if (n_recv > 0 && (!recv_buf || !xq_perm || !xs_perm || !pair_row)) return MOE_ERR_NULL;
    if (n_recv > 0 && (!aligned16(recv_buf) || !aligned16(xq_perm))) return MOE_ERR_ALIGN;
    if (!ws || ws_bytes < moe_ep_workspace_size(shape, n_ranks, n_recv)) return MOE_ERR_WORKSPACE;
    cudaStream_t st = as_stream(stream);
    // the chunk counts and totals live after the plan's mask
    uint8_t* base = static_cast<uint8_t*>(ws) +
                    align_up(sizeof(uint32_t) * std::max(shape->T, 1), 256);
    const int n_chunks = (n_recv + kEpChunk - 1) / kEpChunk;
    int32_t* totals = reinterpret_cast<int32_t*>(base);
    int32_t* chunk_counts = totals + align_up(size_t(E), 64);
    if (cudaMemsetAsync(totals, 0, sizeof(int32_t) * E, st) != cudaSuccess) return MOE_ERR_CUDA;
    if (n_recv > 0) {
        ep_chunk_hist_kernel<<<n_chunks, 256, sizeof(int) * E, st>>>(recv_buf, n_recv, d, K, E,
                                                                   chunk_counts, totals,
                                                                   dev_status);
        if ((rc = check_launch()) != MOE_OK) return rc;
    }
    ep_chunk_scan_kernel<<<E, 256, 0, st>>>(totals, E, n_chunks, chunk_counts, local_offsets);
    if ((rc = check_launch()) != MOE_OK) return rc;
    if (n_recv == 0) return MOE_OK;
    ep_chunk_rank_kernel<<<n_chunks, 32, sizeof(int) * 2 * E, st>>>(
        recv_buf, n_recv, d, K, E, chunk_counts, local_offsets, max_rows, pair_row, dev_status);
    if ((rc = check_launch()) != MOE_OK) return rc;
    ep_copy_rows_kernel<<<warp_grid(n_recv), 256, 0, st>>>(
        recv_buf, n_recv, d, K, pair_row, int64_t(max_rows), reinterpret_cast<uint4*>(xq_perm),
        xs_perm);
    return check_launch();
}

extern "C" MOE_API int moe_ep_partial_combine(const MoeShape* shape, int n_ranks,
                                              const uint8_t* recv_buf, int n_recv,
                                              const int32_t* pair_row, const float* expert_out,
                                              float* back_buf, int* dev_status, void* stream) {
    (void)dev_status;
    int rc = ep_check(shape, n_ranks);
    if (rc != MOE_OK) return rc;
    if (n_recv < 0) return MOE_ERR_SHAPE;
    if (n_recv == 0) return MOE_OK;
    if (!recv_buf || !pair_row || !expert_out || !back_buf) return MOE_ERR_NULL;
    if (!aligned16(expert_out) || !aligned16(back_buf)) return MOE_ERR_ALIGN;
    const int64_t chunks = (shape->d / 4 + 32 * kEpU - 1) / (32 * kEpU);
    ep_partial_combine_kernel<<<warp_grid(int64_t(n_recv) * chunks), 256, 0, as_stream(stream)>>>(
        recv_buf, n_recv, shape->d, shape->topk, pair_row,
        reinterpret_cast<const float4*>(expert_out), reinterpret_cast<float4*>(back_buf));
    return check_launch();
}

extern "C" MOE_API int moe_ep_final_combine(const MoeShape* shape, int n_ranks,
                                            const float* shared_out, const float* back_recv,
                                            const int32_t* send_row, uint16_t* y,
                                            int* dev_status, void* stream) {
    (void)dev_status;
    int rc = ep_check(shape, n_ranks);
    if (rc != MOE_OK) return rc;
    const int T = shape->T;
    if (T == 0) return MOE_OK;
    if (!shared_out || !send_row || !y) return MOE_ERR_NULL;
    if (!aligned16(shared_out) || (back_recv && !aligned16(back_recv)) ||
        (reinterpret_cast<uintptr_t>(y) & 7))
        return MOE_ERR_ALIGN;
    const int64_t chunks = (shape->d / 4 + 32 * kEpU - 1) / (32 * kEpU);
    ep_final_combine_kernel<<<warp_grid(int64_t(T) * chunks), 256, 0, as_stream(stream)>>>(
        reinterpret_cast<const float4*>(shared_out), reinterpret_cast<const float4*>(back_recv),
        T, shape->d, n_ranks, send_row, reinterpret_cast<uint2*>(y));
    return check_launch();
}
