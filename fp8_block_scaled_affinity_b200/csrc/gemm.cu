// Grouped FP8 E4M3 expert GEMM with 1x128 / 128x128 block scales applied on
// the FP32 accumulator ("DeepSeek-V3 Technical Report" notes page, section
// "FP8 mixed precision training": fine-grained quantisation; increased
// accumulation precision, where partial sums are promoted to FP32 every
// N_C = 128 elements of K).  On H800 the promotion moved WGMMA partials to
// CUDA-core registers; here each 128-deep K block is one tcgen05 MMA chain
// into a fresh TMEM buffer, and promotion warps fold it into register FP32
// accumulators with the block's combined scale sa[token] * sb[weight block].
//
// Tile: 128 tokens (the MMA's M side, one token per TMEM lane, so a thread's
// token scale is one register) x BN weight columns (N) x 128 K.
//   BN = 256 (SwiGLU epilogue): the gate (W1) and up (W3) blocks of the same
//     128 features, so a thread holds gate and up of the same (token,
//     feature); 2 TMEM partial buffers, 4 smem stages of 48 KB.
//   BN = 128 (fp32 / bf16 output): one 128-row weight block; 4 TMEM partial
//     buffers (more slack between MMA and promotion), 4 stages of 32 KB; a
//     warp's 32 finished row segments go to a swizzled tile in shared memory
//     and leave as TMA bulk tensor stores (full 128-byte lines, written by
//     the copy engine while the next tile's K loop runs); the rows of a
//     group's ragged last warp are stored directly.
//
// Roles (384 threads, one CTA per SM, persistent over work items):
//   warp 0       TMA producer: token tile (16 KB) + weight tile(s) per K block
//   warp 1       TMEM owner and MMA issuer (one thread)
//   warp 2       scale loader: cp.async of the K block's 128 token scales and
//                the weight-block scales into a small smem ring
//   warp 3       idle (its registers go to the promoters)
//   warps 4-11   promotion + epilogue: warp w reads TMEM lanes 32*(w%4)..+31
//                (its 32 tokens) and one half of the BN columns
#include <cuda.h>
#include <cuda_bf16.h>
#include <mutex>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kThreads = 384;
constexpr int kTileBytes = 128 * 128;            // one 128 x 128 FP8 tile
constexpr int kStages = 4;                       // smem ring of operand stages
constexpr int kParkWarpBytes = 32 * 256;         // one warp's 32 parked rows (fp32 halves)
constexpr int kMaxBufs = 4;
constexpr int kScaleSlots = 16;
constexpr int kMaxGroups = 1040;
constexpr int kBM = 128;                         // tokens per tile
constexpr int kPromoters = 8;                    // promotion warps

template <int BN>
struct Cfg {
    static constexpr int kStageBytes = kTileBytes + BN * 128;  // tokens + weights
    static constexpr int kStages = moe::kStages;
    static constexpr int kRingBytes = kStages * kStageBytes;
    static constexpr int kParkBytes = BN == 128 ? kPromoters * kParkWarpBytes : 0;
    static constexpr int kBufs = 512 / BN;                     // TMEM partial buffers
    static constexpr int kPairs = BN / 4;                      // fp32 pairs per promoter thread
    static_assert(kBufs <= kMaxBufs, "TMEM buffers");
};

struct GemmParams {
    const int32_t* group_offsets;
    int n_groups;
    int max_rows;
    const float* a_scales;  // [nkb, max_rows]
    int k;
    int nkb;
    const float* w_scales;  // [n_groups, n/128, nkb]
    int n;                  // weight rows per group
    int n_ftiles;           // BN-column tiles per group
    int epilogue;
    void* out;
    float* out_scales;
    int* dev_status;
};

struct SharedState {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t tfull[kMaxBufs];
    uint64_t tempty[kMaxBufs];
    uint64_t sfull[kScaleSlots];
    uint64_t sempty[kScaleSlots];
    uint64_t drain;
    uint32_t tmem_base;
    int abort_flag;
    int total_items;
    int goff[kMaxGroups + 1];
    int gstart[kMaxGroups + 1];
    alignas(16) float sa[kScaleSlots][kBM];   // token scales of one K block
    alignas(16) float sb[kScaleSlots][2];     // the weight-block scale(s)
    alignas(16) float red[2][2][kBM];         // [item parity][half][token] amax of h
};

template <int BN>
constexpr size_t smem_bytes() {
    return size_t(Cfg<BN>::kRingBytes) + Cfg<BN>::kParkBytes + sizeof(SharedState) + 1024;
}
static_assert(smem_bytes<256>() <= 232448 && smem_bytes<128>() <= 232448,
              "dynamic shared memory above the sm_100 limit per CTA");

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

// The waiting thread is suspended until the phase completes or about
// kSuspendNs pass, so waiting warps do not take issue slots from the others.
constexpr uint32_t kSuspendNs = 50000;

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "n"(kSuspendNs)
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
        if ((it & 15) == 0) {
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

// 4-byte asynchronous copy global -> shared; src_bytes = 0 writes a zero.
__device__ __forceinline__ void cp_async4(void* dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)),
                 "l"(src), "r"(src_bytes)
                 : "memory");
}

// Arrive on `bar` once this thread's earlier cp.async copies have landed.
__device__ __forceinline__ void cp_async_arrive(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
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

// 32 consecutive TMEM columns of this warp's 32 lanes -> 32 registers; the
// wait for the load is part of the same statement.
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

// 64 consecutive TMEM columns of this warp's 32 lanes -> 64 registers; the
// wait for the load is part of the same statement.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, "
        "%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, "
        "%48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]),
          "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]),
          "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]),
          "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]),
          "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]),
          "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ uint64_t pack2(uint32_t lo, uint32_t hi) {
    uint64_t v;
    asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "r"(lo), "r"(hi));
    return v;
}
__device__ __forceinline__ float2 unpack2(uint64_t v) {
    float2 f;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(f.x), "=f"(f.y) : "l"(v));
    return f;
}
// acc (two fp32 lanes) += p * s, one instruction for two values.
__device__ __forceinline__ void ffma2(uint64_t& acc, uint64_t p, uint64_t s) {
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(p), "l"(s));
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
    int g;      // group
    int f;      // BN-column tile
    int row0;   // first token row
    int ntok;   // valid tokens (<= 128)
};

__device__ __forceinline__ Item decode_item(const SharedState* ss, const GemmParams& p, int item) {
    int lo = 0, hi = p.n_groups;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (ss->gstart[mid] <= item) lo = mid;
        else hi = mid;
    }
    Item it;
    it.g = lo;
    const int local = item - ss->gstart[lo];
    const int rows = ss->goff[lo + 1] - ss->goff[lo];
    const int mtiles = (rows + kBM - 1) / kBM;
    it.f = local / mtiles;
    const int mt = local - it.f * mtiles;
    it.row0 = ss->goff[lo] + mt * kBM;
    it.ntok = min(kBM, rows - mt * kBM);
    return it;
}

// 128-row weight block(s) of a tile: first row inside the stacked
// [n_groups * n, k] matrix and block-row index (for its scales).
template <int BN>
__device__ __forceinline__ void weight_blocks(const GemmParams& p, const Item& w, int& r0, int& r1,
                                              int& b0, int& b1) {
    if (BN == 256) {
        b0 = w.f;                   // gate rows f*128 .. of W1
        b1 = p.n / 256 + w.f;       // up rows (n/2 + f*128) .. of W3
    } else {
        b0 = w.f;
        b1 = w.f;
    }
    r0 = w.g * p.n + b0 * 128;
    r1 = w.g * p.n + b1 * 128;
}

// ================================================= TMA producer (warp 0)
template <int BN>
__device__ __forceinline__ void producer(const GemmParams& p, const CUtensorMap& map_w,
                                         const CUtensorMap& map_a, uint8_t* smem,
                                         SharedState* ss) {
    using C = Cfg<BN>;
    const int lane = threadIdx.x & 31;
    const int total_items = ss->total_items;
    uint32_t it = 0;
    uint32_t issued_mask = 0, issued_parity = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < total_items; item += gridDim.x) {
        const Item w = decode_item(ss, p, item);
        int wr0, wr1, b0, b1;
        weight_blocks<BN>(p, w, wr0, wr1, b0, b1);
        for (int kb = 0; kb < p.nkb; ++kb, ++it) {
            const int s = it % C::kStages;
            const uint32_t par = ((it / C::kStages) & 1u);
            if (lane == 0) ok = mbar_wait(smem_u32(&ss->empty[s]), par ^ 1u, ss, p.dev_status);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            if (lane == 0) {
                uint8_t* st = smem + size_t(s) * C::kStageBytes;
                const uint32_t fb = smem_u32(&ss->full[s]);
                mbar_arrive_expect_tx(fb, uint32_t(C::kStageBytes));
                tma_load_2d(smem_u32(st), &map_a, fb, kb * 128, w.row0);
                tma_load_2d(smem_u32(st + kTileBytes), &map_w, fb, kb * 128, wr0);
                if (BN == 256)
                    tma_load_2d(smem_u32(st + 2 * kTileBytes), &map_w, fb, kb * 128, wr1);
                issued_mask |= 1u << s;
                issued_parity = (issued_parity & ~(1u << s)) | (par << s);
            }
        }
    }
    if (!ok && lane == 0) {
        // let loads already in flight land before the CTA leaves
        for (int s = 0; s < C::kStages; ++s)
            if ((issued_mask >> s) & 1u)
                mbar_wait(smem_u32(&ss->full[s]), (issued_parity >> s) & 1u, ss, nullptr);
    }
    __syncwarp();
}

// ================================================= scale loader (warp 2)
// cp.async of each K block's 128 token scales (kb-major, so they are
// contiguous) and the tile's weight-block scale(s); the copies arrive on
// sfull when they land.
template <int BN>
__device__ __forceinline__ void scale_loader(const GemmParams& p, SharedState* ss) {
    const int lane = threadIdx.x & 31;
    const int total_items = ss->total_items;
    const int nbr = p.n / 128;  // weight block rows per group
    uint32_t cit = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < total_items; item += gridDim.x) {
        const Item w = decode_item(ss, p, item);
        int wr0, wr1, b0, b1;
        weight_blocks<BN>(p, w, wr0, wr1, b0, b1);
        const float* sb0 = p.w_scales + (size_t(w.g) * nbr + b0) * p.nkb;
        const float* sb1 = p.w_scales + (size_t(w.g) * nbr + b1) * p.nkb;
        for (int kb = 0; kb < p.nkb; ++kb, ++cit) {
            const int c = cit % kScaleSlots;
            if (lane == 0)
                ok = mbar_wait(smem_u32(&ss->sempty[c]), ((cit / kScaleSlots) & 1u) ^ 1u, ss,
                               p.dev_status);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            const float* sa = p.a_scales + size_t(kb) * p.max_rows + w.row0;
#pragma unroll
            for (int i = 0; i < kBM / 32; ++i) {
                const int j = lane + 32 * i;
                const bool real = j < w.ntok;  // rows past the group get 0
                cp_async4(&ss->sa[c][j], real ? sa + j : sa, real ? 4u : 0u);
            }
            if (lane == 0) {
                cp_async4(&ss->sb[c][0], sb0 + kb, 4u);
                cp_async4(&ss->sb[c][1], sb1 + kb, 4u);
            }
            cp_async_arrive(smem_u32(&ss->sfull[c]));
        }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncwarp();
}

// ================================================= MMA issuer (warp 1)
template <int BN>
__device__ __forceinline__ void mma_issuer(const GemmParams& p, uint8_t* smem, SharedState* ss,
                                           uint32_t tmem_base) {
    using C = Cfg<BN>;
    const int lane = threadIdx.x & 31;
    const int total_items = ss->total_items;
    if (lane == 0) {
        uint32_t it = 0, tb = 0;
        bool ok = true;
        const uint32_t idesc = idesc_e4m3(128, BN);
        for (int item = blockIdx.x; ok && item < total_items; item += gridDim.x) {
            for (int kb = 0; kb < p.nkb; ++kb, ++it, ++tb) {
                const int s = it % C::kStages;
                const uint32_t buf = tb % C::kBufs;
                const uint32_t tpar = (tb / C::kBufs) & 1u;
                ok = mbar_wait(smem_u32(&ss->tempty[buf]), tpar ^ 1u, ss, p.dev_status);
                if (!ok) break;
                ok = mbar_wait(smem_u32(&ss->full[s]), (it / C::kStages) & 1u, ss, p.dev_status);
                if (!ok) break;
                tc_fence_after();
                const uint32_t st = smem_u32(smem + size_t(s) * C::kStageBytes);
                const uint32_t d = tmem_base + buf * BN;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_e4m3(d, sw128_desc(st + kk * 32), sw128_desc(st + kTileBytes + kk * 32),
                             idesc, kk > 0 ? 1u : 0u);
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

// fp32 / bf16 epilogue: a warp's 32 finished row segments (64 values each)
// are written into its parking tile in shared memory in the 128-byte swizzle
// layout of the output tensor map (16-byte chunk c of row r at c ^ (r % 8)),
// then one lane hands the tile to the TMA engine as bulk tensor stores.  The
// next tile waits until the engine has read the parking tile.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(src), "r"(x), "r"(y)
        : "memory");
}
__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ================================================= promotion + epilogue (warps 4-11)
// Thread (warp w, lane l) owns token row r = 32*(w%4) + l of the tile and
// half h = (w-4)/4 of its columns:
//   BN = 256 (SwiGLU): gate columns [64h, 64h+64) and up columns
//     [128+64h, 128+64h+64) (the same 64 features of W1 and W3);
//   BN = 128: columns [64h, 64h+64) of the single weight block.
template <int BN>
__device__ __forceinline__ void promoter(const GemmParams& p, SharedState* ss, char* park_area,
                                         uint32_t tmem_base, const CUtensorMap* map_o) {
    using C = Cfg<BN>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int total_items = ss->total_items;
    const int q = warp & 3;
    const int half = (warp - 4) >> 2;
    const int r = q * 32 + lane;  // token row inside the tile
    const uint32_t lane_addr = tmem_base + (uint32_t(q * 32) << 16);
    const bool bf16_out = p.epilogue == MOE_EPI_BF16;
    const int c0 = BN == 256 ? half * 64 : half * 64;        // first column of chunk 0
    const int c1 = BN == 256 ? 128 + half * 64 : half * 64;  // first column of chunk 1
    uint32_t tb = 0, cit = 0, parity = 0;
    bool ok = true;
    // this warp's parking tile (swizzled, 1024-byte aligned)
    char* const wpark = park_area + (warp - 4) * kParkWarpBytes;
    for (int item = blockIdx.x; item < total_items; item += gridDim.x, parity ^= 1u) {
        const Item w = decode_item(ss, p, item);
        uint64_t acc2[C::kPairs];  // fp32 accumulator pairs
#pragma unroll
        for (int i = 0; i < C::kPairs; ++i) acc2[i] = 0;
        for (int kb = 0; ok && kb < p.nkb; ++kb, ++tb, ++cit) {
            const uint32_t buf = tb % C::kBufs;
            const int c = cit % kScaleSlots;
            if (lane == 0) {
                ok = mbar_wait(smem_u32(&ss->tfull[buf]), (tb / C::kBufs) & 1u, ss, p.dev_status);
                if (ok) ok = mbar_wait(smem_u32(&ss->sfull[c]), (cit / kScaleSlots) & 1u, ss,
                                       p.dev_status);
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            __syncwarp();
            tc_fence_after();
            const float sa = ss->sa[c][r];
            const float s0 = sa * ss->sb[c][0];
            const float s1 = sa * ss->sb[c][1];
            const uint64_t s0x2 = pack2(__float_as_uint(s0), __float_as_uint(s0));
            const uint64_t s1x2 = pack2(__float_as_uint(s1), __float_as_uint(s1));
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&ss->sempty[c]));  // scales read
            if (BN == 256) {
                uint32_t v[64];
                tmem_ld64(lane_addr + buf * BN + c0, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) ffma2(acc2[i], pack2(v[2 * i], v[2 * i + 1]), s0x2);
                tmem_ld64(lane_addr + buf * BN + c1, v);
                // the partial is in registers: hand the TMEM buffer back to
                // the MMA before the last FMAs
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&ss->tempty[buf]));
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    ffma2(acc2[32 + i], pack2(v[2 * i], v[2 * i + 1]), s1x2);
            } else {
                uint32_t v[32];
                tmem_ld32(lane_addr + buf * BN + c0, v);
#pragma unroll
                for (int i = 0; i < 16; ++i) ffma2(acc2[i], pack2(v[2 * i], v[2 * i + 1]), s0x2);
                tmem_ld32(lane_addr + buf * BN + c0 + 32, v);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&ss->tempty[buf]));
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    ffma2(acc2[16 + i], pack2(v[2 * i], v[2 * i + 1]), s0x2);
            }
        }
        // ---------------- epilogue
        const bool row_ok = r < w.ntok;
        const size_t row = size_t(w.row0) + r;
        if (BN == 128) {
            const int rows_here = w.ntok - q * 32;  // valid rows of this warp's 32
            const int col = w.f * 128 + half * 64;
            if (rows_here >= 32) {
                // the engine has read the previous tile out of the parking tile
                if (lane == 0) bulk_wait_read();
                __syncwarp();
                if (bf16_out) {
                    // one 128-byte box: 64 bf16 per row
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        uint32_t u[4];
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            const float2 f = unpack2(acc2[4 * j + h]);
                            __nv_bfloat162 b2 = __floats2bfloat162_rn(f.x, f.y);
                            u[h] = *reinterpret_cast<uint32_t*>(&b2);
                        }
                        *reinterpret_cast<uint4*>(wpark + lane * 128 + ((j ^ (lane & 7)) * 16)) =
                            make_uint4(u[0], u[1], u[2], u[3]);
                    }
                } else {
                    // two 128-byte boxes: columns [0, 32) and [32, 64) of the half
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float2 a = unpack2(acc2[2 * i]), b = unpack2(acc2[2 * i + 1]);
                        char* box = wpark + (i >> 3) * 4096;
                        *reinterpret_cast<float4*>(box + lane * 128 + (((i & 7) ^ (lane & 7)) * 16)) =
                            make_float4(a.x, a.y, b.x, b.y);
                    }
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    const int y = w.row0 + q * 32;
                    if (bf16_out) {
                        tma_store_2d(map_o, smem_u32(wpark), col, y);
                    } else {
                        tma_store_2d(map_o, smem_u32(wpark), col, y);
                        tma_store_2d(map_o, smem_u32(wpark + 4096), col + 32, y);
                    }
                    bulk_commit();
                }
            } else if (row_ok) {
                // the group's ragged last rows: plain stores, only the valid rows
                if (bf16_out) {
                    uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) +
                                                          row * p.n + col);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        uint32_t u[4];
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            const float2 f = unpack2(acc2[4 * j + h]);
                            __nv_bfloat162 b2 = __floats2bfloat162_rn(f.x, f.y);
                            u[h] = *reinterpret_cast<uint32_t*>(&b2);
                        }
                        dst[j] = make_uint4(u[0], u[1], u[2], u[3]);
                    }
                } else {
                    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + row * p.n + col);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float2 a = unpack2(acc2[2 * i]), b = unpack2(acc2[2 * i + 1]);
                        dst[i] = make_float4(a.x, a.y, b.x, b.y);
                    }
                }
            }
        } else {
            // h = silu(gate) * up for this thread's 64 features, then the
            // 1x128 scale of the token's 128 features (both halves).
            float acc[128];
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                const float2 f = unpack2(acc2[i]);
                acc[2 * i] = f.x;
                acc[2 * i + 1] = f.y;
            }
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                const float g = acc[i];
                // silu(g) = g / (1 + e^-g); fast exp and divide (~1e-6 relative)
                const float hv = __fdividef(g, 1.0f + __expf(-g)) * acc[64 + i];
                acc[i] = hv;
                amax = fmaxf(amax, fabsf(hv));
            }
            ss->red[parity][half][r] = amax;
            named_bar(1, kPromoters * 32);
            amax = fmaxf(amax, ss->red[parity][half ^ 1][r]);
            float scale, inv;
            scale_from_amax(amax, scale, inv);
            if (row_ok) {
                uint4* o = reinterpret_cast<uint4*>(static_cast<uint8_t*>(p.out) + row * (p.n / 2) +
                                                    size_t(w.f) * 128 + half * 64);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    uint32_t u[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int b = 16 * i + 4 * j;
                        const uint32_t lo = e4m3x2(__fmul_rn(acc[b], inv), __fmul_rn(acc[b + 1], inv));
                        const uint32_t hi = e4m3x2(__fmul_rn(acc[b + 2], inv), __fmul_rn(acc[b + 3], inv));
                        u[j] = lo | (hi << 16);
                    }
                    o[i] = make_uint4(u[0], u[1], u[2], u[3]);
                }
                if (half == 0) p.out_scales[size_t(w.f) * p.max_rows + row] = scale;
            }
        }
        // all promotion warps agree on whether to go on
        const bool any_abort = named_bar_or(
            2, kPromoters * 32, !ok || *reinterpret_cast<volatile int*>(&ss->abort_flag));
        if (any_abort) break;
    }
    // every bulk store of this warp has completed before the CTA moves on
    if (BN == 128 && lane == 0) bulk_wait_all();
    __syncwarp();
    tc_fence_before();
}

// ----------------------------------------------------------------- kernel
template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap map_w,
                        const __grid_constant__ CUtensorMap map_a,
                        const __grid_constant__ CUtensorMap map_o, const GemmParams p) {
    using C = Cfg<BN>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    SharedState* ss =
        reinterpret_cast<SharedState*>(smem + size_t(C::kRingBytes) + C::kParkBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- prologue: barriers, TMEM, schedule
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(smem_u32(&ss->full[s]), 1);
            mbar_init(smem_u32(&ss->empty[s]), 1);
        }
        for (int b = 0; b < C::kBufs; ++b) {
            mbar_init(smem_u32(&ss->tfull[b]), 1);
            mbar_init(smem_u32(&ss->tempty[b]), kPromoters);
        }
        for (int c = 0; c < kScaleSlots; ++c) {
            mbar_init(smem_u32(&ss->sfull[c]), 32);
            mbar_init(smem_u32(&ss->sempty[c]), kPromoters);
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
    // group offsets (validated) and an exclusive scan of work items per group
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
                v = ((rows + kBM - 1) / kBM) * p.n_ftiles;
            }
            vals[j] = v;
            sum += v;
        }
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
        set_max_regs_dec<72>();
        if (warp == 0) producer<BN>(p, map_w, map_a, smem, ss);
        else if (warp == 1) mma_issuer<BN>(p, smem, ss, tmem_base);
        else if (warp == 2) scale_loader<BN>(p, ss);
    } else {
        set_max_regs_inc<208>();
        promoter<BN>(p, ss, reinterpret_cast<char*>(smem + C::kRingBytes), tmem_base, &map_o);
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem_base)
                     : "memory");
    }
}

template <int BN>
int launch(const GemmParams& p, const CUtensorMap& mw, const CUtensorMap& ma,
           const CUtensorMap& mo, cudaStream_t st) {
    if (cudaFuncSetAttribute(grouped_gemm_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(smem_bytes<BN>())) != cudaSuccess)
        return MOE_ERR_CUDA;
    grouped_gemm_kernel<BN><<<sm_count(), kThreads, smem_bytes<BN>(), st>>>(mw, ma, mo, p);
    return check_launch();
}

}  // namespace

// ------------------------------------------------------------------ host
// Tensor maps and the device check (declared in common.cuh; the router uses
// them too).
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

// 2D output map over [rows, cols] of fp32 or bf16 (cols contiguous): box = 32 rows x
// 128 bytes, 128-byte swizzle (the layout of the epilogue's parking tiles).
bool make_out_map(CUtensorMap* m, void* base, uint64_t rows, uint64_t cols, bool bf16) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const uint32_t esize = bf16 ? 2 : 4;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * esize};
    cuuint32_t box[2] = {128 / esize, 32};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base,
              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool device_is_sm100() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return false;
    return major == 10;
}

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
    const bool swiglu = epilogue == MOE_EPI_SWIGLU_QUANT;
    p.n_ftiles = swiglu ? n / 256 : n / 128;
    p.epilogue = epilogue;
    p.out = out;
    p.out_scales = out_scales;
    p.dev_status = dev_status;

    CUtensorMap mw, ma, mo;
    if (!make_map(&mw, w, uint64_t(n_groups) * n, uint64_t(k), 128) ||
        !make_map(&ma, a, uint64_t(max_rows), uint64_t(k), 128))
        return MOE_ERR_CUDA;
    if (swiglu) mo = mw;  // unused by the SwiGLU epilogue
    else if (!make_out_map(&mo, out, uint64_t(max_rows), uint64_t(n), epilogue == MOE_EPI_BF16))
        return MOE_ERR_CUDA;
    return swiglu ? launch<256>(p, mw, ma, mo, as_stream(stream))
                  : launch<128>(p, mw, ma, mo, as_stream(stream));
}
