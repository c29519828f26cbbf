// Grouped FP8 E4M3 expert GEMM with 1x128 / 128x128 block scales applied on
// the FP32 accumulator ("DeepSeek-V3 Technical Report" notes page, section
// "FP8 mixed precision training": fine-grained quantisation; increased
// accumulation precision, where partial sums are promoted to FP32 every
// N_C = 128 elements of K).  On H800 the promotion moved WGMMA partials to
// CUDA-core registers; here each 128-deep K block is one tcgen05 MMA chain
// into a fresh TMEM buffer, and promotion warps fold it into register FP32
// accumulators with the block's combined scale sa[token] * sb[weight block].
//
// Layout ("swap AB"): the weight tile is the MMA's M side (128 rows = one
// 128x128 quantisation block row), the tokens are the N side (16..256,
// rounded up to 16), so small expert groups waste no tensor work and a
// weight tile is streamed once per token tile.
//
// Roles (384 threads, one CTA per SM, persistent over work items):
//   warp 0       TMA producer: weight tiles + token tiles into a 4-stage
//                smem ring; combined scales into a small smem ring
//   warp 1       TMEM owner and MMA issuer (one thread)
//   warps 2-3    idle (they give their registers to the promoters)
//   warps 4-11   promotion + epilogue: warp w reads TMEM lanes
//                32*(w%4)..+31 (weight rows) and one half of the columns
//
// Work item = (group g, feature tile f, token tile): NUM_ACC = 2 (SwiGLU)
// computes gate and up rows of the same 128 features into two accumulators
// of up to 128 tokens; NUM_ACC = 1 computes 128 output features for up to
// 256 tokens.  TMEM: 2 partial buffers x 256 columns = all 512 columns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <mutex>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kThreads = 384;
constexpr int kStages = 4;
constexpr int kStageBytes = 48 * 1024;
constexpr int kCombSlots = 8;
constexpr int kMaxGroups = 1040;
constexpr int kTileBytes = 128 * 128;  // one 128 x 128 FP8 tile

struct GemmParams {
    const int32_t* group_offsets;
    int n_groups;
    int max_rows;
    const float* a_scales;  // [nkb, max_rows]
    int k;
    int nkb;
    const float* w_scales;  // [n_groups, n/128, nkb]
    int n;                  // weight rows per group
    int n_feat;             // feature tiles per group
    int epilogue;
    void* out;
    float* out_scales;
    int* dev_status;
};

struct SharedState {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t cfull[kCombSlots];
    uint64_t cempty[kCombSlots];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    int total_items;
    int goff[kMaxGroups + 1];
    int gstart[kMaxGroups + 1];
    alignas(16) float red[2][4][64];
    alignas(16) float inv[2][64];
    alignas(16) float comb[kCombSlots][256];
};

constexpr size_t kSmemBytes = size_t(kStages) * kStageBytes + sizeof(SharedState) + 1024;

// ------------------------------------------------------------- PTX glue
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait: returns false (and raises the CTA's abort flag and the
// device status) when the phase does not complete within kWaitLimitNs, or
// when another role of the CTA has already aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, SharedState* ss,
                                       int* dev_status) {
    if (mbar_try_wait(bar, parity)) return true;
    uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 255) == 0) {
            if (*reinterpret_cast<volatile int*>(&ss->abort_flag)) return false;
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                atomicExch(&ss->abort_flag, 1);
                set_status(dev_status, MOE_DEV_TIMEOUT);
                return false;
            }
        }
    }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// K-major operand tile in shared memory, 128-byte swizzle: rows of 128 bytes
// (one 128-deep K block of E4M3), 8-row atoms 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= uint64_t((saddr & 0x3FFFFu) >> 4);       // start address
    d |= uint64_t(16 >> 4) << 16;                 // leading byte offset (unused here)
    d |= uint64_t(1024 >> 4) << 32;               // stride byte offset: 8 rows x 128 B
    d |= uint64_t(1) << 46;                       // descriptor version for tcgen05
    d |= uint64_t(2) << 61;                       // 128-byte swizzle
    return d;
}

// kind::f8f6f4 instruction descriptor: D fp32, A and B E4M3, both K-major.
__device__ __forceinline__ uint32_t idesc_e4m3(int m, int n) {
    return (1u << 4) | (uint32_t(n >> 3) << 17) | (uint32_t(m >> 4) << 24);
}

__device__ __forceinline__ void mma_e4m3(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

// 32 consecutive TMEM columns of this warp's 32 lanes -> 32 registers,
// waiting for the load to finish.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ uint64_t pack2(uint32_t lo, uint32_t hi) {
    uint64_t v;
    asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "r"(lo), "r"(hi));
    return v;
}
__device__ __forceinline__ void unpack2(uint64_t v, float& lo, float& hi) {
    uint32_t a, b;
    asm("mov.b64 {%0, %1}, %2;" : "=r"(a), "=r"(b) : "l"(v));
    lo = __uint_as_float(a);
    hi = __uint_as_float(b);
}
// acc(2 lanes) += p(2 lanes) * c(2 lanes), one instruction for two floats.
__device__ __forceinline__ void ffma2(uint64_t& acc, uint64_t p, uint64_t c) {
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(p), "l"(c));
}

__device__ __forceinline__ void named_bar(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// Barrier over `count` threads that also ORs a predicate across them.
__device__ __forceinline__ bool named_bar_or(int id, int count, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(uint32_t(pred)), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}

template <int N>
__device__ __forceinline__ void set_max_regs_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void set_max_regs_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// ------------------------------------------------------------- schedule
struct Item {
    int g, f, row0, ntok, nmma;
};

template <int NMAX>
__device__ __forceinline__ Item decode_item(const SharedState* ss, int n_groups, int item) {
    int lo = 0, hi = n_groups;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (ss->gstart[mid] <= item) lo = mid;
        else hi = mid;
    }
    Item it;
    it.g = lo;
    const int local = item - ss->gstart[lo];
    const int rows = ss->goff[lo + 1] - ss->goff[lo];
    const int ntiles = (rows + NMAX - 1) / NMAX;
    it.f = local / ntiles;
    const int tt = local - it.f * ntiles;
    const int base = rows / ntiles, rem = rows - base * ntiles;
    it.ntok = base + (tt < rem ? 1 : 0);
    it.row0 = ss->goff[lo] + tt * base + min(tt, rem);
    it.nmma = max(16, (it.ntok + 15) & ~15);
    return it;
}

// ================================================= TMA producer (warp 0)
template <int NUM_ACC>
__device__ __forceinline__ void producer(const GemmParams& p, const CUtensorMap& map_w,
                                         const CUtensorMap& map_a64, const CUtensorMap& map_a16,
                                         uint8_t* smem, SharedState* ss) {
    constexpr int NMAX = 256 / NUM_ACC;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    (void)warp;
    (void)lane;
    const int G = p.n_groups;
    const int total_items = ss->total_items;
    // ================================================= TMA producer
    uint32_t it = 0, cit = 0;
    uint32_t issued_mask = 0, issued_parity = 0;
    bool ok = true;
    const int nfw = p.n / 128;  // weight block rows per group
    for (int item = blockIdx.x; ok && item < total_items; item += gridDim.x) {
        const Item w = decode_item<NMAX>(ss, G, item);
        const int wrow0 = w.g * p.n + w.f * 128;
        const int wrow1 = wrow0 + p.n / 2;  // up projection (NUM_ACC == 2)
        const uint32_t tx = uint32_t(NUM_ACC * kTileBytes + w.nmma * 128);
        const float* sbw = p.w_scales + (size_t(w.g) * nfw + w.f) * p.nkb;
        const float* sbw1 = p.w_scales + (size_t(w.g) * nfw + w.f + nfw / 2) * p.nkb;
        for (int kb = 0; kb < p.nkb; ++kb, ++it, ++cit) {
            const int s = it % kStages;
            const uint32_t par = ((it / kStages) & 1u);
            if (lane == 0) ok = mbar_wait(smem_u32(&ss->empty[s]), par ^ 1u, ss, p.dev_status);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            if (lane == 0) {
                uint8_t* st = smem + size_t(s) * kStageBytes;
                const uint32_t fb = smem_u32(&ss->full[s]);
                mbar_arrive_expect_tx(fb, tx);
                tma_load_2d(smem_u32(st), &map_w, fb, kb * 128, wrow0);
                if (NUM_ACC == 2) tma_load_2d(smem_u32(st + kTileBytes), &map_w, fb, kb * 128, wrow1);
                uint8_t* bt = st + NUM_ACC * kTileBytes;
                int r = 0;
                for (; r + 64 <= w.nmma; r += 64)
                    tma_load_2d(smem_u32(bt + r * 128), &map_a64, fb, kb * 128, w.row0 + r);
                for (; r < w.nmma; r += 16)
                    tma_load_2d(smem_u32(bt + r * 128), &map_a16, fb, kb * 128, w.row0 + r);
                issued_mask |= 1u << s;
                issued_parity = (issued_parity & ~(1u << s)) | (par << s);
            }
            // combined scales sa[token] * sb[weight block] for this K block
            const int c = cit % kCombSlots;
            const uint32_t cpar = ((cit / kCombSlots) & 1u);
            if (lane == 0) ok = mbar_wait(smem_u32(&ss->cempty[c]), cpar ^ 1u, ss, p.dev_status);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            const float sb0 = __ldg(sbw + kb);
            const float sb1 = NUM_ACC == 2 ? __ldg(sbw1 + kb) : 0.0f;
            const float* sa = p.a_scales + size_t(kb) * p.max_rows + w.row0;
            for (int j = lane; j < w.nmma; j += 32) {
                const float a = j < w.ntok ? __ldg(sa + j) : 0.0f;
                ss->comb[c][j] = a * sb0;
                if (NUM_ACC == 2) ss->comb[c][128 + j] = a * sb1;
            }
            mbar_arrive(smem_u32(&ss->cfull[c]));
        }
    }
    if (!ok && lane == 0) {
        // let loads already in flight land before the CTA leaves
        for (int s = 0; s < kStages; ++s)
            if ((issued_mask >> s) & 1u)
                mbar_wait(smem_u32(&ss->full[s]), (issued_parity >> s) & 1u, ss, nullptr);
    }
    __syncwarp();
}

// ================================================= MMA issuer (warp 1)
template <int NUM_ACC>
__device__ __forceinline__ void mma_issuer(const GemmParams& p, uint8_t* smem, SharedState* ss,
                                           uint32_t tmem_base) {
    constexpr int NMAX = 256 / NUM_ACC;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    (void)warp;
    (void)lane;
    const int G = p.n_groups;
    const int total_items = ss->total_items;
    // ================================================= MMA issuer
    if (lane == 0) {
        uint32_t it = 0, tb = 0;
        bool ok = true;
        for (int item = blockIdx.x; ok && item < total_items; item += gridDim.x) {
            const Item w = decode_item<NMAX>(ss, G, item);
            const uint32_t idesc = idesc_e4m3(128, w.nmma);
            for (int kb = 0; kb < p.nkb; ++kb, ++it, ++tb) {
                const int s = it % kStages;
                const uint32_t buf = tb & 1u;
                ok = mbar_wait(smem_u32(&ss->tempty[buf]), ((tb >> 1) & 1u) ^ 1u, ss, p.dev_status);
                if (!ok) break;
                ok = mbar_wait(smem_u32(&ss->full[s]), (it / kStages) & 1u, ss, p.dev_status);
                if (!ok) break;
                tc_fence_after();
                const uint32_t st = smem_u32(smem + size_t(s) * kStageBytes);
                const uint32_t bt = st + NUM_ACC * kTileBytes;
#pragma unroll
                for (int a = 0; a < NUM_ACC; ++a) {
                    const uint32_t d = tmem_base + buf * 256 + a * 128;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_e4m3(d, sw128_desc(st + a * kTileBytes + kk * 32),
                                 sw128_desc(bt + kk * 32), idesc, kk > 0 ? 1u : 0u);
                }
                mma_commit(smem_u32(&ss->empty[s]));
                mma_commit(smem_u32(&ss->tfull[buf]));
            }
        }
        // all MMAs issued by this thread have completed once drain fires
        mma_commit(smem_u32(&ss->drain));
        mbar_wait(smem_u32(&ss->drain), 0, ss, nullptr);
    }
    __syncwarp();
}

// ================================================= promotion + epilogue (warps 4-11)
template <int NUM_ACC>
__device__ __forceinline__ void promoter(const GemmParams& p, SharedState* ss,
                                         uint32_t tmem_base) {
    constexpr int NMAX = 256 / NUM_ACC;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    (void)warp;
    (void)lane;
    const int G = p.n_groups;
    const int total_items = ss->total_items;
    // ================================================= promotion + epilogue
    const int q = warp & 3;          // TMEM lane quadrant = weight rows 32q..32q+31
    const int half = (warp - 4) >> 2;  // column half
    const uint32_t lane_addr = tmem_base + (uint32_t(q * 32) << 16);
    uint32_t tb = 0, cit = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < total_items; item += gridDim.x) {
        const Item w = decode_item<NMAX>(ss, G, item);
        uint64_t acc[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) acc[i] = 0;
        for (int kb = 0; ok && kb < p.nkb; ++kb, ++tb, ++cit) {
            const uint32_t buf = tb & 1u;
            const int c = cit % kCombSlots;
            if (lane == 0) {
                ok = mbar_wait(smem_u32(&ss->tfull[buf]), (tb >> 1) & 1u, ss, p.dev_status);
                if (ok) ok = mbar_wait(smem_u32(&ss->cfull[c]), (cit / kCombSlots) & 1u, ss,
                                       p.dev_status);
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                // column (token) offset of this 32-column chunk inside its accumulator
                const int rc = NUM_ACC == 2 ? half * 64 + (ch & 1) * 32 : half * 128 + ch * 32;
                const int a = NUM_ACC == 2 ? (ch >> 1) : 0;
                if (rc >= w.nmma) continue;
                uint32_t r[32];
                tmem_ld32(lane_addr + buf * 256 + a * 128 + rc, r);
                const float4* cs = reinterpret_cast<const float4*>(&ss->comb[c][a * 128 + rc]);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float4 cv = cs[i];
                    ffma2(acc[ch * 16 + 2 * i], pack2(r[4 * i], r[4 * i + 1]),
                          pack2(__float_as_uint(cv.x), __float_as_uint(cv.y)));
                    ffma2(acc[ch * 16 + 2 * i + 1], pack2(r[4 * i + 2], r[4 * i + 3]),
                          pack2(__float_as_uint(cv.z), __float_as_uint(cv.w)));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(smem_u32(&ss->tempty[buf]));
                mbar_arrive(smem_u32(&ss->cempty[c]));
            }
        }
        // ---------------- epilogue
        const int feat = q * 32 + lane;  // row inside the 128-row weight tile
        if (NUM_ACC == 1) {
            const size_t ld = size_t(p.n);
            const int col0 = w.f * 128 + feat;
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                float v0, v1;
                unpack2(acc[i], v0, v1);
                const int j = half * 128 + 2 * i;
                if (p.epilogue == MOE_EPI_F32) {
                    float* o = static_cast<float*>(p.out);
                    if (j < w.ntok) o[size_t(w.row0 + j) * ld + col0] = v0;
                    if (j + 1 < w.ntok) o[size_t(w.row0 + j + 1) * ld + col0] = v1;
                } else {
                    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out);
                    if (j < w.ntok) o[size_t(w.row0 + j) * ld + col0] = __float2bfloat16_rn(v0);
                    if (j + 1 < w.ntok)
                        o[size_t(w.row0 + j + 1) * ld + col0] = __float2bfloat16_rn(v1);
                }
            }
        } else {
            // h = silu(gate) * up for 64 tokens (this half), then 1x128
            // quantisation over the tile's 128 features (4 quadrant warps).
            float h[64];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                float g0, g1, u0, u1;
                unpack2(acc[i], g0, g1);
                unpack2(acc[32 + i], u0, u1);
                h[2 * i] = __fmul_rn(__fdiv_rn(g0, 1.0f + expf(-g0)), u0);
                h[2 * i + 1] = __fmul_rn(__fdiv_rn(g1, 1.0f + expf(-g1)), u1);
            }
            // column maxima of |h| over this warp's 32 lanes: after the
            // butterfly, lane l holds the max of column (32*b + l).
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = fabsf(h[32 * b + i]);
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) {
                    const bool upper = (lane & o) != 0;
#pragma unroll
                    for (int i = 0; i < o; ++i) {
                        const float send = upper ? v[i] : v[i + o];
                        const float keep = upper ? v[i + o] : v[i];
                        v[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, o));
                    }
                }
                ss->red[half][q][32 * b + lane] = v[0];
            }
            named_bar(1 + half, 128);
            if (q == 0) {
#pragma unroll
                for (int b = 0; b < 2; ++b) {
                    const int jj = 32 * b + lane;
                    float amax = fmaxf(fmaxf(ss->red[half][0][jj], ss->red[half][1][jj]),
                                       fmaxf(ss->red[half][2][jj], ss->red[half][3][jj]));
                    float scale, inv;
                    scale_from_amax(amax, scale, inv);
                    ss->inv[half][jj] = inv;
                    const int j = half * 64 + jj;
                    if (j < w.ntok) p.out_scales[size_t(w.f) * p.max_rows + w.row0 + j] = scale;
                }
            }
            named_bar(1 + half, 128);
            uint8_t* o = static_cast<uint8_t*>(p.out);
            const size_t ld = size_t(p.n / 2);
            const int col0 = w.f * 128 + feat;
#pragma unroll
            for (int i = 0; i < 64; i += 2) {
                const int j = half * 64 + i;
                const uint16_t c2 = e4m3x2(__fmul_rn(h[i], ss->inv[half][i]),
                                           __fmul_rn(h[i + 1], ss->inv[half][i + 1]));
                if (j < w.ntok) o[size_t(w.row0 + j) * ld + col0] = uint8_t(c2 & 0xFF);
                if (j + 1 < w.ntok) o[size_t(w.row0 + j + 1) * ld + col0] = uint8_t(c2 >> 8);
            }
        }
        // all warps of this half agree on whether to go on
        const bool any_abort =
            named_bar_or(3 + half, 128, !ok || *reinterpret_cast<volatile int*>(&ss->abort_flag));
        if (any_abort) break;
    }
    tc_fence_before();
}

// ----------------------------------------------------------------- kernel
template <int NUM_ACC>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap map_w,
                        const __grid_constant__ CUtensorMap map_a64,
                        const __grid_constant__ CUtensorMap map_a16, const GemmParams p) {
    constexpr int NMAX = 256 / NUM_ACC;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    SharedState* ss = reinterpret_cast<SharedState*>(smem + size_t(kStages) * kStageBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- prologue: barriers, TMEM, schedule
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&ss->full[s]), 1);
            mbar_init(smem_u32(&ss->empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&ss->tfull[b]), 1);
            mbar_init(smem_u32(&ss->tempty[b]), 8);
        }
        for (int c = 0; c < kCombSlots; ++c) {
            mbar_init(smem_u32(&ss->cfull[c]), 32);
            mbar_init(smem_u32(&ss->cempty[c]), 8);
        }
        mbar_init(smem_u32(&ss->drain), 1);
        ss->abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                         smem_u32(&ss->tmem_base))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // group offsets and an exclusive scan of work items per group
    const int G = p.n_groups;
    int bad = 0;
    for (int i = threadIdx.x; i <= G; i += kThreads) {
        const int v = p.group_offsets[i];
        ss->goff[i] = v;
        if (v < 0 || v > p.max_rows || (i > 0 && v < p.group_offsets[i - 1])) bad = 1;
    }
    // offsets that are negative, decreasing or past max_rows: no work at all
    if (__syncthreads_or(bad)) {
        if (threadIdx.x == 0) set_status(p.dev_status, MOE_DEV_BAD_INPUT);
        for (int i = threadIdx.x; i <= G; i += kThreads) ss->goff[i] = 0;
        __syncthreads();
    }
    {
        constexpr int PER = (kMaxGroups + kThreads) / kThreads;  // entries per thread
        int vals[PER];
        int sum = 0;
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            const int g = threadIdx.x * PER + j;
            int v = 0;
            if (g < G) {
                const int rows = ss->goff[g + 1] - ss->goff[g];
                v = rows > 0 ? ((rows + NMAX - 1) / NMAX) * p.n_feat : 0;
            }
            vals[j] = v;
            sum += v;
        }
        // block exclusive scan of per-thread sums (reuse gstart as scratch)
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += n;
        }
        __shared__ int wsum[kThreads / 32];
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        int before = 0, total = 0;
        for (int w = 0; w < kThreads / 32; ++w) {
            if (w < warp) before += wsum[w];
            total += wsum[w];
        }
        int run = before + incl - sum;
#pragma unroll
        for (int j = 0; j < PER; ++j) {
            const int g = threadIdx.x * PER + j;
            if (g <= G) ss->gstart[g] = run;
            run += vals[j];
        }
        if (threadIdx.x == 0) ss->total_items = total;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = ss->tmem_base;

    if (warp < 4) {
        set_max_regs_dec<56>();
        if (warp == 0) producer<NUM_ACC>(p, map_w, map_a64, map_a16, smem, ss);
        else if (warp == 1) mma_issuer<NUM_ACC>(p, smem, ss, tmem_base);
    } else {
        set_max_regs_inc<224>();
        promoter<NUM_ACC>(p, ss, tmem_base);
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem_base)
                     : "memory");
    }
}


// ------------------------------------------------------------------ host
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// 2D uint8 map over [rows, cols] (cols contiguous), box = [box_rows, 128].
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols};
    cuuint32_t box[2] = {128, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

bool device_is_sm100() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return false;
    return major == 10;
}

template <int NUM_ACC>
int launch(const GemmParams& p, const CUtensorMap& mw, const CUtensorMap& m64,
           const CUtensorMap& m16, cudaStream_t st) {
    if (cudaFuncSetAttribute(grouped_gemm_kernel<NUM_ACC>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(kSmemBytes)) != cudaSuccess)
        return MOE_ERR_CUDA;
    grouped_gemm_kernel<NUM_ACC><<<sm_count(), kThreads, kSmemBytes, st>>>(mw, m64, m16, p);
    return check_launch();
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" MOE_API int moe_grouped_gemm_fp8(int n_groups, const int32_t* group_offsets,
                                            int max_rows, const uint8_t* a,
                                            const float* a_scales, int k, const uint8_t* w,
                                            const float* w_scales, int n, int epilogue,
                                            void* out, float* out_scales, int* dev_status,
                                            void* stream) {
    if (n_groups < 1 || n_groups > kMaxGroups || max_rows < 0 || k <= 0 || k % 128 || n <= 0 ||
        n % 128)
        return MOE_ERR_SHAPE;
    if (epilogue != MOE_EPI_F32 && epilogue != MOE_EPI_BF16 && epilogue != MOE_EPI_SWIGLU_QUANT)
        return MOE_ERR_ARG;
    if (epilogue == MOE_EPI_SWIGLU_QUANT && n % 256) return MOE_ERR_SHAPE;
    if (!group_offsets || !w || !w_scales || !out) return MOE_ERR_NULL;
    if (epilogue == MOE_EPI_SWIGLU_QUANT && !out_scales) return MOE_ERR_NULL;
    if (max_rows == 0) return MOE_OK;
    if (!a || !a_scales) return MOE_ERR_NULL;
    if (!aligned16(a) || !aligned16(w) || !aligned16(out)) return MOE_ERR_ALIGN;
    if (int64_t(n_groups) * n > INT32_MAX) return MOE_ERR_SHAPE;
    if (!device_is_sm100()) return MOE_ERR_DEVICE;

    GemmParams p;
    p.group_offsets = group_offsets;
    p.n_groups = n_groups;
    p.max_rows = max_rows;
    p.a_scales = a_scales;
    p.k = k;
    p.nkb = k / 128;
    p.w_scales = w_scales;
    p.n = n;
    p.n_feat = epilogue == MOE_EPI_SWIGLU_QUANT ? n / 256 : n / 128;
    p.epilogue = epilogue;
    p.out = out;
    p.out_scales = out_scales;
    p.dev_status = dev_status;

    CUtensorMap mw, m64, m16;
    if (!make_map(&mw, w, uint64_t(n_groups) * n, uint64_t(k), 128) ||
        !make_map(&m64, a, uint64_t(max_rows), uint64_t(k), 64) ||
        !make_map(&m16, a, uint64_t(max_rows), uint64_t(k), 16))
        return MOE_ERR_CUDA;
    cudaStream_t st = as_stream(stream);
    if (epilogue == MOE_EPI_SWIGLU_QUANT) return launch<2>(p, mw, m64, m16, st);
    return launch<1>(p, mw, m64, m16, st);
}
