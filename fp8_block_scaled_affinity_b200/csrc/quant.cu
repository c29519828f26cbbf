// Online FP8 E4M3 quantisation: 1x128 activation tiles and 128x128 weight
// blocks ("DeepSeek-V3 Technical Report" notes page, section "FP8 mixed
// precision training": fine-grained quantisation, online max-abs scaling,
// E4M3 for every tensor).  Both are single coalesced HBM passes with 16-byte
// vector loads and stores.
#include "common.cuh"

namespace moe {
namespace {

// One 1x128 tile per 16 threads; each thread owns 8 consecutive bf16 values
// (one 16-byte load, one 8-byte store) of kActUnroll tiles at a time, whose
// loads are all issued before any is used, so each thread keeps several
// loads in flight.  Grid-strides over tiles.
constexpr int kActUnroll = 4;

// POW2: power-of-two scales written as UE8M0 bytes to sf (scales unused).
template <bool POW2>
__global__ void __launch_bounds__(256) quant_act_1x128_kernel(
    const uint4* __restrict__ x, int64_t rows, int64_t cols, uint2* __restrict__ q,
    float* __restrict__ scales, uint8_t* __restrict__ sf, int kb_major) {
    const int64_t tiles_per_row = cols >> 7;
    const int64_t n_tiles = rows * tiles_per_row;
    const int sub = threadIdx.x & 15;
    // Both half-warps iterate together (the shuffles span the full warp; the
    // stride is even, so the two tiles of a warp stay a pair); a half-warp
    // past the last tile computes on zeros and stores nothing.
    int64_t tile = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 4;
    const int64_t tile_stride = (int64_t(gridDim.x) * blockDim.x) >> 4;
    for (; (tile & ~int64_t(1)) < n_tiles; tile += kActUnroll * tile_stride) {
        uint4 w[kActUnroll];
        int64_t vec[kActUnroll], r[kActUnroll], t[kActUnroll];
#pragma unroll
        for (int u = 0; u < kActUnroll; ++u) {
            const int64_t tt = tile + u * tile_stride;
            const bool valid = tt < n_tiles;
            r[u] = valid ? tt / tiles_per_row : -1;
            t[u] = valid ? tt - r[u] * tiles_per_row : 0;
            vec[u] = valid ? (r[u] * cols + (t[u] << 7)) / 8 + sub : 0;
            w[u] = valid ? __ldcs(x + vec[u]) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kActUnroll; ++u) {
            float v[8] = {bf16_lo(w[u].x), bf16_hi(w[u].x), bf16_lo(w[u].y), bf16_hi(w[u].y),
                          bf16_lo(w[u].z), bf16_hi(w[u].z), bf16_lo(w[u].w), bf16_hi(w[u].w)};
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
            for (int o = 8; o >= 1; o >>= 1)
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            float scale, inv;
            int e = 0;
            if (POW2) {
                e = pow2_exponent(amax);
                inv = pow2_inverse(e);
                scale = 0.0f;
            } else {
                scale_from_amax(amax, scale, inv);
            }
            uint32_t c0 = e4m3x2(__fmul_rn(v[0], inv), __fmul_rn(v[1], inv));
            uint32_t c1 = e4m3x2(__fmul_rn(v[2], inv), __fmul_rn(v[3], inv));
            uint32_t c2 = e4m3x2(__fmul_rn(v[4], inv), __fmul_rn(v[5], inv));
            uint32_t c3 = e4m3x2(__fmul_rn(v[6], inv), __fmul_rn(v[7], inv));
            if (r[u] < 0) continue;
            q[vec[u]] = make_uint2(c0 | (c1 << 16), c2 | (c3 << 16));
            if (sub == 0) {
                const int64_t at = kb_major ? t[u] * rows + r[u] : r[u] * tiles_per_row + t[u];
                if (POW2) sf[at] = uint8_t(e + 127);
                else scales[at] = scale;
            }
        }
    }
}

// One 128x128 block per CTA iteration, 512 threads; thread i owns a quarter
// row (32 values = 4 x 16-byte loads).  Block amax via warp shuffles + smem.
// The next block's vectors are loaded into registers before the current
// block is reduced and stored, so every thread keeps its loads in flight.
constexpr int kWThreads = 512;

template <bool POW2>
__global__ void __launch_bounds__(kWThreads) quant_w_128x128_kernel(
    const uint4* __restrict__ w, int64_t rows, int64_t cols, uint4* __restrict__ q,
    float* __restrict__ scales, uint8_t* __restrict__ sf) {
    constexpr int kWarps = kWThreads / 32;
    __shared__ float warp_max[2][kWarps];
    const int64_t bc = cols >> 7;
    const int64_t n_blocks = (rows >> 7) * bc;
    const int row = threadIdx.x >> 2, quarter = threadIdx.x & 3;
    auto base_of = [&](int64_t b) {  // in 16-byte vectors (8 values)
        const int64_t bi = b / bc, bj = b - bi * bc;
        return ((bi * 128 + row) * cols + bj * 128 + quarter * 32) / 8;
    };
    int64_t b = blockIdx.x;
    uint4 v[4];
    if (b < n_blocks) {
        const int64_t base = base_of(b);
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = __ldcs(w + base + i);
    }
    for (int it = 0; b < n_blocks; b += gridDim.x, ++it) {
        const int64_t bn = b + gridDim.x;
        uint4 nv[4];
        if (bn < n_blocks) {
            const int64_t base = base_of(bn);
#pragma unroll
            for (int i = 0; i < 4; ++i) nv[i] = __ldcs(w + base + i);
        }
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            amax = fmaxf(amax, fabsf(bf16_lo(v[i].x)));
            amax = fmaxf(amax, fabsf(bf16_hi(v[i].x)));
            amax = fmaxf(amax, fabsf(bf16_lo(v[i].y)));
            amax = fmaxf(amax, fabsf(bf16_hi(v[i].y)));
            amax = fmaxf(amax, fabsf(bf16_lo(v[i].z)));
            amax = fmaxf(amax, fabsf(bf16_hi(v[i].z)));
            amax = fmaxf(amax, fabsf(bf16_lo(v[i].w)));
            amax = fmaxf(amax, fabsf(bf16_hi(v[i].w)));
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        // two slots alternate, so one barrier per block suffices
        float* wm = warp_max[it & 1];
        if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = amax;
        __syncthreads();
        amax = wm[0];
#pragma unroll
        for (int i = 1; i < kWarps; ++i) amax = fmaxf(amax, wm[i]);
        float scale, inv;
        int e = 0;
        if (POW2) {
            e = pow2_exponent(amax);
            inv = pow2_inverse(e);
            scale = 0.0f;
        } else {
            scale_from_amax(amax, scale, inv);
        }
        const int64_t bi = b / bc, bj = b - bi * bc;
        const int64_t qbase = ((bi * 128 + row) * cols + bj * 128 + quarter * 32) / 16;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            uint32_t o[4];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const uint4 s = v[2 * i + j];
                uint32_t a0 = e4m3x2(__fmul_rn(bf16_lo(s.x), inv), __fmul_rn(bf16_hi(s.x), inv));
                uint32_t a1 = e4m3x2(__fmul_rn(bf16_lo(s.y), inv), __fmul_rn(bf16_hi(s.y), inv));
                uint32_t a2 = e4m3x2(__fmul_rn(bf16_lo(s.z), inv), __fmul_rn(bf16_hi(s.z), inv));
                uint32_t a3 = e4m3x2(__fmul_rn(bf16_lo(s.w), inv), __fmul_rn(bf16_hi(s.w), inv));
                o[2 * j] = a0 | (a1 << 16);
                o[2 * j + 1] = a2 | (a3 << 16);
            }
            __stcs(q + qbase + i, make_uint4(o[0], o[1], o[2], o[3]));
        }
        if (threadIdx.x == 0) {
            if (POW2) sf[b] = uint8_t(e + 127);
            else scales[b] = scale;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = nv[i];
    }
}

}  // namespace
}  // namespace moe

using namespace moe;

namespace moe {
namespace {

int launch_act(const uint16_t* x, int64_t rows, int64_t cols, uint8_t* q, float* scales,
               uint8_t* sf, int kb_major, void* stream) {
    const int64_t threads = rows * (cols / 128) * 16;
    int64_t blocks = (threads + 256 * kActUnroll - 1) / (256 * kActUnroll);
    const int64_t cap = int64_t(sm_count()) * 8;
    if (blocks > cap) blocks = cap;
    if (sf)
        quant_act_1x128_kernel<true><<<unsigned(blocks), 256, 0, as_stream(stream)>>>(
            reinterpret_cast<const uint4*>(x), rows, cols, reinterpret_cast<uint2*>(q), scales, sf,
            kb_major);
    else
        quant_act_1x128_kernel<false><<<unsigned(blocks), 256, 0, as_stream(stream)>>>(
            reinterpret_cast<const uint4*>(x), rows, cols, reinterpret_cast<uint2*>(q), scales, sf,
            kb_major);
    return check_launch();
}

int launch_w(const uint16_t* w, int64_t rows, int64_t cols, uint8_t* q, float* scales,
             uint8_t* sf, void* stream) {
    const int64_t n_blocks = (rows / 128) * (cols / 128);
    int64_t grid = n_blocks;
    const int64_t cap = int64_t(sm_count()) * 4;  // 4 CTAs of 512 threads per SM
    if (grid > cap) grid = cap;
    if (sf)
        quant_w_128x128_kernel<true><<<unsigned(grid), kWThreads, 0, as_stream(stream)>>>(
            reinterpret_cast<const uint4*>(w), rows, cols, reinterpret_cast<uint4*>(q), scales, sf);
    else
        quant_w_128x128_kernel<false><<<unsigned(grid), kWThreads, 0, as_stream(stream)>>>(
            reinterpret_cast<const uint4*>(w), rows, cols, reinterpret_cast<uint4*>(q), scales, sf);
    return check_launch();
}

}  // namespace
}  // namespace moe

extern "C" MOE_API int fp8_quant_act_1x128(const uint16_t* x, int64_t rows, int64_t cols,
                                           uint8_t* q, float* scales, int scales_kb_major,
                                           int* dev_status, void* stream) {
    (void)dev_status;
    if (rows < 0 || cols < 0 || cols % 128) return MOE_ERR_SHAPE;
    if (rows == 0 || cols == 0) return MOE_OK;
    if (!x || !q || !scales) return MOE_ERR_NULL;
    if (!aligned16(x) || !aligned16(q) || (reinterpret_cast<uintptr_t>(scales) & 3))
        return MOE_ERR_ALIGN;
    if (scales_kb_major != 0 && scales_kb_major != 1) return MOE_ERR_ARG;
    return launch_act(x, rows, cols, q, scales, nullptr, scales_kb_major, stream);
}

extern "C" MOE_API int fp8_quant_w_128x128(const uint16_t* w, int64_t rows, int64_t cols,
                                           uint8_t* q, float* scales, int* dev_status,
                                           void* stream) {
    (void)dev_status;
    if (rows < 0 || cols < 0 || rows % 128 || cols % 128) return MOE_ERR_SHAPE;
    if (rows == 0 || cols == 0) return MOE_OK;
    if (!w || !q || !scales) return MOE_ERR_NULL;
    if (!aligned16(w) || !aligned16(q) || (reinterpret_cast<uintptr_t>(scales) & 3))
        return MOE_ERR_ALIGN;
    return launch_w(w, rows, cols, q, scales, nullptr, stream);
}

extern "C" MOE_API int fp8_quant_act_1x128_ue8m0(const uint16_t* x, int64_t rows, int64_t cols,
                                                 uint8_t* q, uint8_t* sf, int sf_kb_major,
                                                 int* dev_status, void* stream) {
    (void)dev_status;
    if (rows < 0 || cols < 0 || cols % 128) return MOE_ERR_SHAPE;
    if (rows == 0 || cols == 0) return MOE_OK;
    if (!x || !q || !sf) return MOE_ERR_NULL;
    if (!aligned16(x) || !aligned16(q)) return MOE_ERR_ALIGN;
    if (sf_kb_major != 0 && sf_kb_major != 1) return MOE_ERR_ARG;
    return launch_act(x, rows, cols, q, nullptr, sf, sf_kb_major, stream);
}

extern "C" MOE_API int fp8_quant_w_128x128_ue8m0(const uint16_t* w, int64_t rows, int64_t cols,
                                                 uint8_t* q, uint8_t* sf, int* dev_status,
                                                 void* stream) {
    (void)dev_status;
    if (rows < 0 || cols < 0 || rows % 128 || cols % 128) return MOE_ERR_SHAPE;
    if (rows == 0 || cols == 0) return MOE_OK;
    if (!w || !q || !sf) return MOE_ERR_NULL;
    if (!aligned16(w) || !aligned16(q)) return MOE_ERR_ALIGN;
    return launch_w(w, rows, cols, q, nullptr, sf, stream);
}
