// Grouped FP8 E4M3 expert GEMM with 1x128 / 128x128 block scales applied on
// the FP32 accumulator ("DeepSeek-V3 Technical Report" notes page, section
// "FP8 mixed precision training": fine-grained quantisation; increased
// accumulation precision, where partial sums are promoted to FP32 every
// N_C = 128 elements of K).  On H800 the promotion moved WGMMA partials to
// CUDA-core registers; here each 128-deep K block is one tcgen05 MMA chain
// into a fresh TMEM buffer, and promotion warps fold it into register FP32
// accumulators with the block's combined scale sa[token] * sb[weight block].
//
// Each CTA owns 128 tokens (the MMA's M side, one token per TMEM lane, so a
// thread's token scale is one register) and, per K block, a TMEM partial of
// 128 x C columns (C = 256; 128 for fp32/bf16 output whose width is not a
// multiple of 256).  The 256 columns are two 128-row weight blocks: the gate
// (W1) and up (W3) blocks of the same 128 features for the SwiGLU epilogue,
// two neighbouring blocks of the output otherwise.
//
// Single CTAs (cta_group::1, the default) load both weight blocks
// themselves.  CTA pairs (cta_group::2, MOEFP8_GEMM_PAIR=1): a cluster of
// two CTAs on two SMs runs one M = 256, N = 256 MMA per 32-deep K step; each
// CTA loads its own 128 tokens and ONE of the two weight blocks, so every
// weight byte crosses L2 -> SM once per 256 tokens instead of once per 128.
// The leader (rank 0) issues the MMAs; both CTAs' TMA loads complete on the
// leader's stage barrier, and the MMA commits arrive on both CTAs' barriers.
// gemm_pair_units picks the form.
//
// Token boxes: the TMA box of a CTA's tokens is 128, 64, 32 or 16 rows (the
// smallest that holds its valid rows; none when it has none), so ragged
// tails and tiny groups do not pull 128 rows through L2.  Shared-memory rows
// past the box hold stale codes; they feed only TMEM lanes whose tokens are
// discarded.
//
// Roles (384 threads, one CTA per SM, persistent over work items; a pair
// shares its items):
//   warp 0       TMA producer
//   warp 1       TMEM owner; in the leader, the MMA issuer (one thread)
//   warp 2       scale loader: cp.async of the K block's 128 token scales and
//                the two weight-block scales into a small smem ring
//   warp 3       idle (its registers go to the promoters)
//   warps 4-11   promotion + epilogue: warp w reads TMEM lanes 32*(w%4)..+31
//                (its 32 tokens) and one half of the C columns
#include <cuda.h>
#include <cuda_bf16.h>
#include <algorithm>
#include <cstdlib>
#include <mutex>

#include "common.cuh"

namespace moe {
namespace {

constexpr int kThreads = 384;
constexpr int kTileBytes = 128 * 128;            // one 128 x 128 FP8 tile
constexpr int kBoxBytes = 4096;                  // one 32-row x 128-byte output box
constexpr int kMaxBufs = 4;
constexpr int kMaxStages = 6;
constexpr int kScaleSlots = 16;
constexpr int kMaxGroups = 1040;
constexpr int kBM = 128;                         // tokens per CTA tile
constexpr int kPromoters = 8;                    // promotion warps
constexpr int kABoxes = 4;                       // token boxes of 128, 64, 32, 16 rows
constexpr int kTokenTilesFirst = 16;             // groups up to this many token tiles: token tiles fastest

template <bool PAIR, bool SWIGLU, bool WIDE>
struct Cfg {
    static_assert(WIDE || !(PAIR || SWIGLU), "pairs and SwiGLU use 256-column partials");
    static constexpr int kAccCols = WIDE ? 256 : 128;              // output columns per item
    // One MMA chain per K block into one kAccCols-column TMEM buffer.  (Two
    // N = 128 chains into four 128-column buffers halve how long a buffer is
    // held, but measured slower on B200: eight N = 128 MMAs and two commits
    // per K block cost more issue time than the 512 cycles the block's MMAs
    // take.)
    static constexpr int kChains = 1;                              // MMA chains per K block
    static_assert(kChains == 1, "the promotion waits on the stage barrier of its K block");
    static constexpr int kBufCols = kAccCols / kChains;            // TMEM columns per buffer
    static constexpr int kBufs = 512 / kBufCols;                   // TMEM partial buffers
    static constexpr int kWRows = PAIR ? 128 : kAccCols;           // weight rows this CTA loads
    static constexpr int kStageBytes = kTileBytes + kWRows * 128;  // tokens + weights
    // single CTAs with fp32/bf16 output and 256 columns: 48 KB stages next to
    // the parking tiles leave room for three
    static constexpr int kStages = (PAIR && SWIGLU) ? 6 : (!PAIR && !SWIGLU && WIDE) ? 3 : 4;
    static constexpr int kRingBytes = kStages * kStageBytes;
    // output boxes parked per warp at a time (one where the operand ring is
    // largest)
    static constexpr int kParkBoxes = SWIGLU ? 0 : (!PAIR && WIDE) ? 1 : 2;
    static constexpr int kParkBytes = kPromoters * kParkBoxes * kBoxBytes;
    static constexpr int kPairs = kAccCols / 4;                    // fp32 pairs per promoter thread
    static constexpr int kItemRows = PAIR ? 2 * kBM : kBM;         // tokens per work item
    static constexpr int kMmaM = PAIR ? 256 : 128;
    static constexpr int kCtas = PAIR ? 2 : 1;
    static_assert(kBufs <= kMaxBufs && kStages <= kMaxStages, "ring sizes");
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
    int n_ftiles;           // column tiles per group
    int epilogue;
    void* out;
    float* out_scales;
    int* dev_status;
    uint64_t wait_limit_ns;  // bound of every wait (kWaitLimitNs unless overridden)
    int fault;               // FaultKind injected from the host (kFaultNone normally)
    // weight matrix of each group (nullable: group g uses matrix g); lets
    // several groups share one expert's weights (redundant experts)
    const int32_t* group_weight;
    int n_weights;           // weight matrices in w (== n_groups without an index)
    // block-scaled (UE8M0) form only
    const uint8_t* a_sf;     // [nkb, max_rows] scale bytes of the tokens' 1x128 tiles
    const uint8_t* w_sf;     // [n_groups, n/128, nkb] scale bytes of the weight blocks
    uint8_t* out_sf;         // SwiGLU: [n/256, max_rows] scale bytes of h
};

// Token tensor maps, one per box height (128, 64, 32, 16 rows).
struct AMaps {
    CUtensorMap m[kABoxes];
};

struct SharedState {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t tfull[kMaxBufs];
    uint64_t tempty[kMaxBufs];
    uint64_t sfull[kScaleSlots];
    uint64_t sempty[kScaleSlots];
    uint64_t drain;
    uint64_t wait_limit;     // ns
    uint32_t tmem_base;
    int abort_flag;
    uint32_t peer_abort;     // cluster address of the peer CTA's abort_flag (0: no peer)
    int total_items;
    int goff[kMaxGroups + 1];
    int gstart[kMaxGroups + 1];
    alignas(16) float sa[kScaleSlots][kBM];   // token scales of one K block
    alignas(16) float sb[kScaleSlots][2];     // the two weight-block scales
    alignas(16) float red[2][2][kBM];         // [item parity][half][token] amax of h
};

template <bool PAIR, bool SWIGLU, bool WIDE>
constexpr size_t smem_bytes() {
    using C = Cfg<PAIR, SWIGLU, WIDE>;
    return size_t(C::kRingBytes) + C::kParkBytes + sizeof(SharedState) + 1024;
}
static_assert(smem_bytes<false, false, false>() <= 232448 &&
                  smem_bytes<false, false, true>() <= 232448 &&
                  smem_bytes<false, true, true>() <= 232448 &&
                  smem_bytes<true, false, true>() <= 232448 &&
                  smem_bytes<true, true, true>() <= 232448,
              "dynamic shared memory above the sm_100 limit per CTA");

// ------------------------------------------------------------- PTX glue
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_index() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_count() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}
// Address of the same shared-memory object in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
// Every thread of both CTAs of the cluster.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
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
// Arrive on a barrier of any CTA of the cluster (cluster address).  The
// data it guards is TMEM, ordered by tcgen05 fences, so CTA-scope release
// semantics suffice.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cbar) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cbar) : "memory");
}

// Wait forms.  kSuspend: the waiting thread is suspended until the phase
// completes or about kSuspendNs pass, so waiting warps do not take issue
// slots from the others (single CTAs: every arrival is local).  kPoll: the
// same without the time hint; kSpin: test_wait, never suspends (the MMA
// issuer of a CTA pair, whose barriers also receive the peer's arrivals).
constexpr uint32_t kSuspendNs = 50000;
enum WaitForm { kSuspend = 0, kPoll = 1, kSpin = 2 };
// waits on barriers that a peer CTA also signals
template <bool PAIR> constexpr int kRemoteWait = PAIR ? kPoll : kSuspend;
template <bool PAIR> constexpr int kIssuerWait = PAIR ? kSpin : kSuspend;

template <int FORM>
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    if (FORM == kSuspend)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(bar), "r"(parity), "n"(kSuspendNs)
            : "memory");
    else if (FORM == kPoll)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
    return ok != 0;
}

// Raise this CTA's abort flag (and the peer's, for a CTA pair).
__device__ __forceinline__ void raise_abort(SharedState* ss) {
    atomicExch(&ss->abort_flag, 1);
    if (ss->peer_abort)
        asm volatile("st.relaxed.cluster.shared::cluster.u32 [%0], %1;" ::"r"(ss->peer_abort),
                     "r"(1)
                     : "memory");
}

// Bounded wait: returns false (and raises the abort flags and the device
// status) when the phase does not complete within the launch's wait limit,
// or when another role of the CTA (or of its peer) has already aborted.
template <int FORM = kSuspend>
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, SharedState* ss,
                                          int* dev_status) {
    if (mbar_try_wait<FORM>(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    const uint64_t limit = ss->wait_limit;
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait<FORM>(bar, parity)) return true;
        if ((it & 15) == 0) {
            if (*reinterpret_cast<volatile int*>(&ss->abort_flag)) return false;
            if (globaltimer_ns() - t0 > limit) {
                raise_abort(ss);
                set_status(dev_status, MOE_DEV_TIMEOUT);
                return false;
            }
        }
    }
}

// Waits for work already in flight (TMA loads into this CTA's shared memory,
// MMAs into its TMEM) before the CTA leaves: unlike mbar_wait it goes on
// after an abort, but it still gives up after the wait limit.
__device__ __forceinline__ bool mbar_quiesce(uint32_t bar, uint32_t parity, SharedState* ss,
                                             int* dev_status) {
    if (mbar_try_wait<kPoll>(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    const uint64_t limit = ss->wait_limit;
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait<kPoll>(bar, parity)) return true;
        if ((it & 15) == 0 && globaltimer_ns() - t0 > limit) {
            set_status(dev_status, MOE_DEV_TIMEOUT);
            return false;
        }
    }
}

// 2D tile load global -> this CTA's shared memory, completing on `bar`.
// PAIR: the .cta_group::2 form, whose barrier may be the leader CTA's
// (a cluster address).  No multicast.
template <bool PAIR>
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y) {
    if (PAIR)
        asm volatile(
            "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
            " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
            "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
            : "memory");
    else
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

// TMEM allocation of all 512 columns (both CTAs of a pair allocate together).
template <bool PAIR>
__device__ __forceinline__ void tmem_alloc_all(uint32_t dst_smem) {
    if (PAIR) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                         dst_smem)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    } else {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                         dst_smem)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
}
template <bool PAIR>
__device__ __forceinline__ void tmem_free_all(uint32_t base) {
    if (PAIR)
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, 512;" ::"r"(base)
                     : "memory");
    else
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(base)
                     : "memory");
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

// PAIR: one M = 256 MMA over both CTAs (A rows 0-127 and B rows 0-127 from
// the leader's shared memory, rows 128-255 from the peer's, same offsets).
template <bool PAIR>
__device__ __forceinline__ void mma_e4m3(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
    if (PAIR)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// Arrive on `bar` of this CTA once the MMAs issued so far have completed.
template <bool PAIR>
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    if (PAIR)
        asm volatile(
            "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
            : "memory");
    else
        asm volatile(
            "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
            : "memory");
}
// As mma_commit, arriving on the barrier at the same offset in both CTAs of
// a pair.
template <bool PAIR>
__device__ __forceinline__ void mma_commit_both(uint32_t bar) {
    if (PAIR)
        asm volatile(
            "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
            " [%0], %1;" ::"r"(bar),
            "h"(uint16_t(3))
            : "memory");
    else
        mma_commit<false>(bar);
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
    int f;      // column tile
    int row0;   // first token row of the item (of the pair's 256 for a CTA pair)
    int rows;   // rows of the group from row0 on (may exceed the item)
};

template <int ITEM_ROWS>
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
    const int mtiles = (rows + ITEM_ROWS - 1) / ITEM_ROWS;
    // Order inside a group.  Small groups (a few token tiles, the common
    // case): token tiles fastest, so the tiles that read one weight tile run
    // side by side and the weight tile crosses HBM once.  Large groups (the
    // hot experts of a skewed batch, up to 128 token tiles): column tiles
    // fastest, so the CTAs running together share a few token tiles and walk
    // the expert's weight tiles (29 MB at most, kept in L2), and the token
    // rows cross HBM once instead of once per column tile.
    int mt;
    if (mtiles <= kTokenTilesFirst) {
        it.f = local / mtiles;
        mt = local - it.f * mtiles;
    } else {
        mt = local / p.n_ftiles;
        it.f = local - mt * p.n_ftiles;
    }
    it.row0 = ss->goff[lo] + mt * ITEM_ROWS;
    it.rows = rows - mt * ITEM_ROWS;
    return it;
}

// Weight matrix of group g (the group itself unless an index is given; an
// out-of-range index falls back to matrix 0 and is reported).
__device__ __forceinline__ int weight_of(const GemmParams& p, int g) {
    if (!p.group_weight) return g;
    const int wi = __ldg(&p.group_weight[g]);
    if (wi < 0 || wi >= p.n_weights) {
        set_status(p.dev_status, MOE_DEV_BAD_INPUT);
        return 0;
    }
    return wi;
}

// Valid tokens of CTA `rank` in an item (0..128).
__device__ __forceinline__ int cta_tokens(const Item& w, int rank) {
    return max(0, min(kBM, w.rows - kBM * rank));
}

// Token box for n valid rows: index into AMaps (128, 64, 32, 16 rows) and
// its bytes; n == 0 loads nothing.
__device__ __forceinline__ int box_index(int n) {
    return n > 64 ? 0 : n > 32 ? 1 : n > 16 ? 2 : 3;
}
__device__ __forceinline__ uint32_t box_bytes(int n) {
    return n == 0 ? 0u : uint32_t(kTileBytes >> box_index(n));
}

// The two 128-row weight blocks of a column tile (block-row indices inside
// one group's [n, k] matrix): their scales go to sb[0] and sb[1], and a CTA
// of a pair loads block b[rank].
template <bool PAIR, bool SWIGLU, bool WIDE>
__device__ __forceinline__ void weight_blocks(const GemmParams& p, const Item& w, int& b0,
                                              int& b1) {
    if (SWIGLU) {
        b0 = w.f;                // gate rows f*128 .. of W1
        b1 = p.n / 256 + w.f;    // up rows (n/2 + f*128) .. of W3
    } else if (WIDE) {
        b0 = 2 * w.f;
        b1 = 2 * w.f + 1;
    } else {
        b0 = w.f;
        b1 = w.f;
    }
}

// ================================================= TMA producer (warp 0)
template <bool PAIR, bool SWIGLU, bool WIDE>
__device__ __forceinline__ void producer(const GemmParams& p, const CUtensorMap* map_w,
                                         const AMaps& maps_a, uint8_t* smem, SharedState* ss,
                                         int rank, int unit, int units) {
    using C = Cfg<PAIR, SWIGLU, WIDE>;
    const int lane = threadIdx.x & 31;
    const int total_items = ss->total_items;
    uint32_t it = 0;
    uint32_t issued_mask = 0, issued_parity = 0;
    bool ok = true;
    for (int item = unit; ok && item < total_items; item += units) {
        const Item w = decode_item<C::kItemRows>(ss, p, item);
        int b0, b1;
        weight_blocks<PAIR, SWIGLU, WIDE>(p, w, b0, b1);
        const int n0 = cta_tokens(w, 0);
        const int n1 = PAIR ? cta_tokens(w, 1) : 0;
        const int my_n = rank ? n1 : n0;
        const CUtensorMap* map_a = &maps_a.m[box_index(my_n)];
        const int a_y = w.row0 + kBM * rank;
        // bytes landing on the stage barrier: every CTA's tokens and weights
        const uint32_t tx = box_bytes(n0) + box_bytes(n1) + uint32_t(C::kCtas * C::kWRows * 128);
        const int wg = weight_of(p, w.g);
        const int wr_mine = wg * p.n + (rank ? b1 : b0) * 128;
        const int wr_second = wg * p.n + b1 * 128;  // single CTA, 256 columns: block b1
        for (int kb = 0; kb < p.nkb; ++kb, ++it) {
            const int s = it % C::kStages;
            const uint32_t par = ((it / C::kStages) & 1u);
            if (lane == 0)
                ok = mbar_wait<kRemoteWait<PAIR>>(smem_u32(&ss->empty[s]), par ^ 1u, ss,
                                                  p.dev_status);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            // injected fault: the first stage is never loaded, so the MMA
            // issuer's wait on it runs out (single CTAs only)
            if (!PAIR && p.fault == kFaultGemmProducer && it == 0) continue;
            if (lane == 0) {
                uint8_t* st = smem + size_t(s) * C::kStageBytes;
                const uint32_t local_full = smem_u32(&ss->full[s]);
                const uint32_t fb = PAIR ? mapa(local_full, 0) : local_full;
                if (rank == 0) mbar_arrive_expect_tx(local_full, tx);
                if (my_n > 0) tma_load_2d<PAIR>(smem_u32(st), map_a, fb, kb * 128, a_y);
                tma_load_2d<PAIR>(smem_u32(st + kTileBytes), map_w, fb, kb * 128, wr_mine);
                if (!PAIR && WIDE)
                    tma_load_2d<PAIR>(smem_u32(st + 2 * kTileBytes), map_w, fb, kb * 128,
                                      wr_second);
                issued_mask |= 1u << s;
                issued_parity = (issued_parity & ~(1u << s)) | (par << s);
            }
        }
    }
    if (!ok && lane == 0 && rank == 0) {
        // let loads already in flight land before the CTA leaves (the stage
        // barriers of a pair are the leader's)
        for (int s = 0; s < C::kStages; ++s)
            if ((issued_mask >> s) & 1u)
                mbar_quiesce(smem_u32(&ss->full[s]), (issued_parity >> s) & 1u, ss, nullptr);
    }
    __syncwarp();
}

// ================================================= scale loader (warp 2)
// cp.async of each K block's 128 token scales (kb-major, so they are
// contiguous) and the tile's two weight-block scales; the copies arrive on
// sfull when they land.
template <bool PAIR, bool SWIGLU, bool WIDE>
__device__ __forceinline__ void scale_loader(const GemmParams& p, SharedState* ss, int rank,
                                             int unit, int units) {
    using C = Cfg<PAIR, SWIGLU, WIDE>;
    const int lane = threadIdx.x & 31;
    const int total_items = ss->total_items;
    const int nbr = p.n / 128;  // weight block rows per group
    uint32_t cit = 0;
    bool ok = true;
    for (int item = unit; ok && item < total_items; item += units) {
        const Item w = decode_item<C::kItemRows>(ss, p, item);
        int b0, b1;
        weight_blocks<PAIR, SWIGLU, WIDE>(p, w, b0, b1);
        const int my_n = cta_tokens(w, rank);
        const int my_row0 = w.row0 + kBM * rank;
        const int wg = weight_of(p, w.g);
        const float* sb0 = p.w_scales + (size_t(wg) * nbr + b0) * p.nkb;
        const float* sb1 = p.w_scales + (size_t(wg) * nbr + b1) * p.nkb;
        for (int kb = 0; kb < p.nkb; ++kb, ++cit) {
            const int c = cit % kScaleSlots;
            if (lane == 0)
                ok = mbar_wait(smem_u32(&ss->sempty[c]), ((cit / kScaleSlots) & 1u) ^ 1u, ss,
                               p.dev_status);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            const float* sa = p.a_scales + size_t(kb) * p.max_rows + my_row0;
#pragma unroll
            for (int i = 0; i < kBM / 32; ++i) {
                const int j = lane + 32 * i;
                const bool real = j < my_n;  // rows past the group get 0
                cp_async4(&ss->sa[c][j], real ? sa + j : p.a_scales, real ? 4u : 0u);
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

// ================================================= MMA issuer (warp 1 of the leader)
template <bool PAIR, bool SWIGLU, bool WIDE>
__device__ __forceinline__ void mma_issuer(const GemmParams& p, uint8_t* smem, SharedState* ss,
                                           uint32_t tmem_base, int unit, int units) {
    using C = Cfg<PAIR, SWIGLU, WIDE>;
    const int lane = threadIdx.x & 31;
    const int total_items = ss->total_items;
    if (lane == 0) {
        uint32_t it = 0, tb = 0;
        bool ok = true;
        const uint32_t idesc = idesc_e4m3(C::kMmaM, C::kBufCols);
        for (int item = unit; ok && item < total_items; item += units) {
            for (int kb = 0; ok && kb < p.nkb; ++kb, ++it) {
                const int s = it % C::kStages;
                ok = mbar_wait<kIssuerWait<PAIR>>(smem_u32(&ss->full[s]), (it / C::kStages) & 1u,
                                                   ss, p.dev_status);
                if (!ok) break;
                tc_fence_after();
                const uint32_t st = smem_u32(smem + size_t(s) * C::kStageBytes);
#pragma unroll
                for (int c = 0; c < C::kChains; ++c, ++tb) {
                    const uint32_t buf = tb % C::kBufs;
                    const uint32_t tpar = (tb / C::kBufs) & 1u;
                    ok = mbar_wait<kIssuerWait<PAIR>>(smem_u32(&ss->tempty[buf]), tpar ^ 1u, ss,
                                                       p.dev_status);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t d = tmem_base + buf * C::kBufCols;
                    const uint32_t b0 = st + kTileBytes + c * kTileBytes;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_e4m3<PAIR>(d, sw128_desc(st + kk * 32), sw128_desc(b0 + kk * 32), idesc,
                                       kk > 0 ? 1u : 0u);
                    // one commit per K block: its completion frees the
                    // stage for the producer AND hands the partial to the
                    // promotion warps (who wait on the same barrier)
                    mma_commit_both<PAIR>(smem_u32(&ss->empty[s]));
                }
            }
        }
        // all MMAs issued by this thread have completed once drain fires
        // (also after an abort: they write TMEM, which is freed at the end)
        mma_commit<PAIR>(smem_u32(&ss->drain));
        mbar_quiesce(smem_u32(&ss->drain), 0, ss, nullptr);
    }
    __syncwarp();
}

// fp32 / bf16 epilogue: a warp's 32 finished row segments are written into
// its parking tile in shared memory in the 128-byte swizzle layout of the
// output tensor map (16-byte chunk c of row r at c ^ (r % 8)), one or two
// 4 KB boxes at a time, then one lane hands them to the TMA engine as bulk
// tensor stores.  Before the tile is rewritten, the engine must have read it.
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

__device__ __forceinline__ uint32_t bf16x2_bits(float2 f) {
    __nv_bfloat162 b2 = __floats2bfloat162_rn(f.x, f.y);
    return *reinterpret_cast<uint32_t*>(&b2);
}

// Write this thread's NP fp32 pairs (one row, NP*2 consecutive columns
// from `col`) of the warp's 32 rows: through the parking tile and bulk
// tensor stores when all 32 rows are valid, else direct stores of valid rows.
template <int NP, int R>
__device__ __forceinline__ void store_rows(const GemmParams& p, const uint64_t (&acc2)[NP],
                                           char* wpark, const CUtensorMap* map_o, int lane,
                                           int rows_here, size_t row, int y0, int col) {
    const bool bf16_out = p.epilogue == MOE_EPI_BF16;
    if (rows_here >= 32) {
        if (bf16_out) {
            // boxes of 64 bf16 (32 pairs); R per round
            constexpr int kBoxes = NP / 32;
#pragma unroll
            for (int r0 = 0; r0 < kBoxes; r0 += R) {
                if (lane == 0) bulk_wait_read();
                __syncwarp();
#pragma unroll
                for (int b = r0; b < r0 + R && b < kBoxes; ++b) {
                    char* box = wpark + (b - r0) * kBoxBytes;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int q0 = 32 * b + 4 * j;
                        *reinterpret_cast<uint4*>(box + lane * 128 + ((j ^ (lane & 7)) * 16)) =
                            make_uint4(bf16x2_bits(unpack2(acc2[q0])),
                                       bf16x2_bits(unpack2(acc2[q0 + 1])),
                                       bf16x2_bits(unpack2(acc2[q0 + 2])),
                                       bf16x2_bits(unpack2(acc2[q0 + 3])));
                    }
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
#pragma unroll
                    for (int b = r0; b < r0 + R && b < kBoxes; ++b)
                        tma_store_2d(map_o, smem_u32(wpark + (b - r0) * kBoxBytes), col + 64 * b,
                                     y0);
                    bulk_commit();
                }
            }
        } else {
            // boxes of 32 fp32 (16 pairs); R per round
            constexpr int kBoxes = NP / 16;
#pragma unroll
            for (int r0 = 0; r0 < kBoxes; r0 += R) {
                if (lane == 0) bulk_wait_read();
                __syncwarp();
#pragma unroll
                for (int b = r0; b < r0 + R; ++b) {
                    char* box = wpark + (b - r0) * kBoxBytes;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float2 a = unpack2(acc2[16 * b + 2 * j]);
                        const float2 c = unpack2(acc2[16 * b + 2 * j + 1]);
                        *reinterpret_cast<float4*>(box + lane * 128 + ((j ^ (lane & 7)) * 16)) =
                            make_float4(a.x, a.y, c.x, c.y);
                    }
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
#pragma unroll
                    for (int b = r0; b < r0 + R; ++b)
                        tma_store_2d(map_o, smem_u32(wpark + (b - r0) * kBoxBytes), col + 32 * b,
                                     y0);
                    bulk_commit();
                }
            }
        }
    } else if (lane < rows_here) {
        // the group's ragged last rows: plain stores, only the valid rows
        if (bf16_out) {
            uint4* dst =
                reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + row * p.n + col);
#pragma unroll
            for (int j = 0; j < NP / 4; ++j)
                dst[j] = make_uint4(bf16x2_bits(unpack2(acc2[4 * j])),
                                    bf16x2_bits(unpack2(acc2[4 * j + 1])),
                                    bf16x2_bits(unpack2(acc2[4 * j + 2])),
                                    bf16x2_bits(unpack2(acc2[4 * j + 3])));
        } else {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + row * p.n + col);
#pragma unroll
            for (int i = 0; i < NP / 2; ++i) {
                const float2 a = unpack2(acc2[2 * i]), c = unpack2(acc2[2 * i + 1]);
                dst[i] = make_float4(a.x, a.y, c.x, c.y);
            }
        }
    }
}

// ================================================= promotion + epilogue (warps 4-11)
// Thread (warp w, lane l) owns token row r = 32*(w%4) + l of its CTA's 128
// and half h = (w-4)/4 of the partial's columns:
//   SwiGLU: gate columns [64h, 64h+64) and up columns [128+64h, 128+64h+64)
//     (the same 64 features of W1 and W3);
//   fp32 / bf16, C = 256: columns [128h, 128h+128) (weight block h);
//   fp32 / bf16, C = 128: columns [64h, 64h+64) of the single weight block.
template <bool PAIR, bool SWIGLU, bool WIDE>
__device__ __forceinline__ void promoter(const GemmParams& p, SharedState* ss, char* park_area,
                                         uint32_t tmem_base, const CUtensorMap* map_o, int rank,
                                         int unit, int units) {
    using C = Cfg<PAIR, SWIGLU, WIDE>;
    constexpr bool kWide = C::kAccCols == 256;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int total_items = ss->total_items;
    const int q = warp & 3;
    const int half = (warp - 4) >> 2;
    const int r = q * 32 + lane;  // token row inside the CTA's tile
    const uint32_t lane_addr = tmem_base + (uint32_t(q * 32) << 16);
    // TMEM columns of the two loads per K block and the weight block of each
    int c0, c1, sel0, sel1;
    if (SWIGLU) {
        c0 = 64 * half; c1 = 128 + 64 * half; sel0 = 0; sel1 = 1;
    } else if (kWide) {
        c0 = 128 * half; c1 = 128 * half + 64; sel0 = half; sel1 = half;
    } else {
        c0 = 64 * half; c1 = 64 * half + 32; sel0 = 0; sel1 = 0;
    }
    uint32_t tb = 0, cit = 0, parity = 0;
    bool ok = true;
    // this warp's parking tile (swizzled, 1024-byte aligned)
    char* const wpark = park_area + (warp - 4) * (C::kParkBoxes * kBoxBytes);
    for (int item = unit; item < total_items; item += units, parity ^= 1u) {
        const Item w = decode_item<C::kItemRows>(ss, p, item);
        uint64_t acc2[C::kPairs];  // fp32 accumulator pairs
#pragma unroll
        for (int i = 0; i < C::kPairs; ++i) acc2[i] = 0;
        for (int kb = 0; ok && kb < p.nkb; ++kb, ++tb, ++cit) {
            const uint32_t buf = tb % C::kBufs;
            const int c = cit % kScaleSlots;
            if (lane == 0) {
                // the K block's MMAs have completed: the stage barrier the
                // producer refills on (the stage cannot complete again before
                // this wait: its next K block needs this warp's release of
                // the TMEM buffer one block later)
                ok = mbar_wait<kRemoteWait<PAIR>>(smem_u32(&ss->empty[tb % C::kStages]),
                                                   (tb / C::kStages) & 1u, ss, p.dev_status);
                if (ok) ok = mbar_wait(smem_u32(&ss->sfull[c]), (cit / kScaleSlots) & 1u, ss,
                                       p.dev_status);
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            __syncwarp();
            tc_fence_after();
            const float sa = ss->sa[c][r];
            const float s0 = sa * ss->sb[c][sel0];
            const float s1 = sa * ss->sb[c][sel1];
            const uint64_t s0x2 = pack2(__float_as_uint(s0), __float_as_uint(s0));
            const uint64_t s1x2 = pack2(__float_as_uint(s1), __float_as_uint(s1));
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&ss->sempty[c]));  // scales read
            const uint32_t tbase = lane_addr + buf * C::kBufCols;
            const uint32_t tempty = smem_u32(&ss->tempty[buf]);
            if (kWide) {
                uint32_t v[64];
                tmem_ld64(tbase + c0, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) ffma2(acc2[i], pack2(v[2 * i], v[2 * i + 1]), s0x2);
                tmem_ld64(tbase + c1, v);
                // the partial is in registers: hand the TMEM buffer back to
                // the MMA (the leader's barrier) before the last FMAs
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (PAIR) mbar_arrive_cluster(mapa(tempty, 0));
                    else mbar_arrive(tempty);
                }
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    ffma2(acc2[32 + i], pack2(v[2 * i], v[2 * i + 1]), s1x2);
            } else {
                uint32_t v[32];
                tmem_ld32(tbase + c0, v);
#pragma unroll
                for (int i = 0; i < 16; ++i) ffma2(acc2[i], pack2(v[2 * i], v[2 * i + 1]), s0x2);
                tmem_ld32(tbase + c1, v);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(tempty);
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    ffma2(acc2[16 + i], pack2(v[2 * i], v[2 * i + 1]), s1x2);
            }
        }
        // ---------------- epilogue
        const int my_n = cta_tokens(w, rank);
        const int my_row0 = w.row0 + kBM * rank;
        const bool row_ok = r < my_n;
        const size_t row = size_t(my_row0) + r;
        if (!SWIGLU) {
            constexpr int kCols = C::kAccCols / 2;  // this thread's columns
            store_rows<C::kPairs, (C::kParkBoxes > 0 ? C::kParkBoxes : 1)>(
                p, acc2, wpark, map_o, lane, my_n - q * 32, row,
                                  my_row0 + q * 32, w.f * C::kAccCols + half * kCols);
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
    if (!SWIGLU && lane == 0) bulk_wait_all();
    __syncwarp();
    tc_fence_before();
}

// ----------------------------------------------------------------- kernel
template <bool PAIR, bool SWIGLU, bool WIDE>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap map_w,
                        const __grid_constant__ AMaps maps_a,
                        const __grid_constant__ CUtensorMap map_o, const GemmParams p) {
    using C = Cfg<PAIR, SWIGLU, WIDE>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    SharedState* ss =
        reinterpret_cast<SharedState*>(smem + size_t(C::kRingBytes) + C::kParkBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // a CTA pair works on one item at a time; a single CTA is its own unit
    const int rank = PAIR ? int(cluster_rank()) : 0;
    const int unit = PAIR ? int(cluster_index()) : int(blockIdx.x);
    const int units = PAIR ? int(cluster_count()) : int(gridDim.x);

    // ---- prologue: barriers, TMEM, schedule
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(smem_u32(&ss->full[s]), 1);
            mbar_init(smem_u32(&ss->empty[s]), 1);
        }
        for (int b = 0; b < C::kBufs; ++b) {
            mbar_init(smem_u32(&ss->tfull[b]), 1);
            mbar_init(smem_u32(&ss->tempty[b]), kPromoters * C::kCtas);
        }
        for (int c = 0; c < kScaleSlots; ++c) {
            mbar_init(smem_u32(&ss->sfull[c]), 32);
            mbar_init(smem_u32(&ss->sempty[c]), kPromoters);
        }
        mbar_init(smem_u32(&ss->drain), 1);
        ss->wait_limit = p.wait_limit_ns;
        ss->abort_flag = 0;
        ss->peer_abort = PAIR ? mapa(smem_u32(&ss->abort_flag), uint32_t(rank ^ 1)) : 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) tmem_alloc_all<PAIR>(smem_u32(&ss->tmem_base));
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
                v = ((rows + C::kItemRows - 1) / C::kItemRows) * p.n_ftiles;
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
    // the peer's barriers are initialised before anyone signals them
    if (PAIR) cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = ss->tmem_base;

    if (warp < 4) {
        set_max_regs_dec<72>();
        if (warp == 0) producer<PAIR, SWIGLU, WIDE>(p, &map_w, maps_a, smem, ss, rank, unit, units);
        else if (warp == 1 && rank == 0)
            mma_issuer<PAIR, SWIGLU, WIDE>(p, smem, ss, tmem_base, unit, units);
        else if (warp == 2) scale_loader<PAIR, SWIGLU, WIDE>(p, ss, rank, unit, units);
    } else {
        set_max_regs_inc<208>();
        promoter<PAIR, SWIGLU, WIDE>(p, ss, reinterpret_cast<char*>(smem + C::kRingBytes), tmem_base,
                               &map_o, rank, unit, units);
    }

    __syncthreads();
    // neither CTA of a pair leaves (or frees TMEM) while the other may still
    // signal its barriers or the leader's MMAs may still write its TMEM
    if (PAIR) cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_free_all<PAIR>(tmem_base);
    }
}

// ============================================== block-scaled form (UE8M0 scales)
// A numerically different option beside the pages' recipe: with power-of-two
// scales (UE8M0 bytes: exponent + 127) the tensor core applies the scales
// itself (tcgen05.mma kind::mxf8f6f4.block_scale, one scale per 32 elements
// of K; a 1x128 tile or 128x128 block repeats its scale over four of them),
// so a K block needs no promotion and one TMEM accumulator serves the whole
// K loop of an item.  Roles: warp 0 TMA producer (tokens + both weight
// blocks of the 256 columns); warp 2 builds each stage's scale chunks in
// shared memory (128 rows x 4 scales per 512 bytes: the 32-bit word of row m
// = 32 m1 + m0 at byte 16 m0 + 4 m1, its four bytes the scales of K
// elements 0-31, ..., 96-127); warp 1 copies them into TMEM (tcgen05.cp
// 32x128b.warpx4) and issues the MMAs; warps 4-11 move the finished
// accumulator out at the end of an item and run the epilogue.
template <bool SWIGLU>
struct MxCfg {
    static constexpr int kStages = SWIGLU ? 4 : 3;
    static constexpr int kStageBytes = kTileBytes + 256 * 128;  // tokens + two weight blocks
    static constexpr int kRingBytes = kStages * kStageBytes;
    static constexpr int kSfStage = 3 * 512;                    // A chunk, two B chunks
    static constexpr int kSfBytes = kStages * kSfStage;
    static constexpr int kParkBoxes = SWIGLU ? 0 : 1;
    static constexpr int kParkBytes = kPromoters * kParkBoxes * kBoxBytes;
    static constexpr int kSfCol = 256;                          // TMEM column of stage 0's scales
    static_assert(kStages <= kMaxStages && kStages <= kScaleSlots, "ring sizes");
};
template <bool SWIGLU>
constexpr size_t mx_smem_bytes() {
    using C = MxCfg<SWIGLU>;
    return size_t(C::kRingBytes) + C::kParkBytes + C::kSfBytes + sizeof(SharedState) + 1024;
}
static_assert(mx_smem_bytes<false>() <= 232448 && mx_smem_bytes<true>() <= 232448,
              "dynamic shared memory above the sm_100 limit per CTA");

// Shared-memory descriptor of a scale chunk for tcgen05.cp: K-major without
// swizzle, 8-row x 16-byte core matrices 128 bytes apart along the rows.
__device__ __forceinline__ uint64_t sf_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= uint64_t((saddr & 0x3FFFFu) >> 4);
    d |= uint64_t(128 >> 4) << 16;
    d |= uint64_t(128 >> 4) << 32;
    d |= uint64_t(1) << 46;
    return d;
}
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
                 : "memory");
}
// kind::mxf8f6f4 block-scaled instruction descriptor: E4M3 x E4M3, UE8M0
// scales, fp32 D, K-major; the scale byte of each operand is selected by
// sf_id (also carried in bits 30-31 of the scale TMEM addresses).
__device__ __forceinline__ uint32_t idesc_mx(int m, int n, uint32_t sf_id) {
    return (sf_id << 4) | (uint32_t(n >> 3) << 17) | (1u << 23) | (uint32_t(m >> 4) << 24) |
           (sf_id << 29);
}
__device__ __forceinline__ void mma_mx(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate, uint32_t sfa, uint32_t sfb) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb));
}

template <bool SWIGLU>
__device__ __forceinline__ void mx_producer(const GemmParams& p, const CUtensorMap* map_w,
                                            const AMaps& maps_a, uint8_t* smem, SharedState* ss,
                                            int unit, int units) {
    using C = MxCfg<SWIGLU>;
    const int lane = threadIdx.x & 31;
    const int total_items = ss->total_items;
    uint32_t it = 0, issued_mask = 0, issued_parity = 0;
    bool ok = true;
    for (int item = unit; ok && item < total_items; item += units) {
        const Item w = decode_item<kBM>(ss, p, item);
        int b0, b1;
        weight_blocks<false, SWIGLU, true>(p, w, b0, b1);
        const int n0 = cta_tokens(w, 0);
        const CUtensorMap* map_a = &maps_a.m[box_index(n0)];
        const uint32_t tx = box_bytes(n0) + uint32_t(256 * 128);
        for (int kb = 0; kb < p.nkb; ++kb, ++it) {
            const int s = it % C::kStages;
            const uint32_t par = (it / C::kStages) & 1u;
            if (lane == 0) ok = mbar_wait(smem_u32(&ss->empty[s]), par ^ 1u, ss, p.dev_status);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            if (lane == 0) {
                uint8_t* st = smem + size_t(s) * C::kStageBytes;
                const uint32_t fb = smem_u32(&ss->full[s]);
                mbar_arrive_expect_tx(fb, tx);
                if (n0 > 0) tma_load_2d<false>(smem_u32(st), map_a, fb, kb * 128, w.row0);
                tma_load_2d<false>(smem_u32(st + kTileBytes), map_w, fb, kb * 128,
                                   w.g * p.n + b0 * 128);
                tma_load_2d<false>(smem_u32(st + 2 * kTileBytes), map_w, fb, kb * 128,
                                   w.g * p.n + b1 * 128);
                issued_mask |= 1u << s;
                issued_parity = (issued_parity & ~(1u << s)) | (par << s);
            }
        }
    }
    if (!ok && lane == 0)
        for (int s = 0; s < C::kStages; ++s)
            if ((issued_mask >> s) & 1u)
                mbar_quiesce(smem_u32(&ss->full[s]), (issued_parity >> s) & 1u, ss, nullptr);
    __syncwarp();
}

// warp 2: the stage's scale chunks (tokens, weight block 0, weight block 1),
// loaded once the stage is free.  (Loading them four K blocks ahead into
// registers measured 8-50% slower on B200.)
template <bool SWIGLU>
__device__ __forceinline__ void mx_scale_loader(const GemmParams& p, uint8_t* sf_area,
                                                SharedState* ss, int unit, int units) {
    using C = MxCfg<SWIGLU>;
    const int lane = threadIdx.x & 31;
    const int total_items = ss->total_items;
    const int nbr = p.n / 128;
    uint32_t it = 0;
    bool ok = true;
    for (int item = unit; ok && item < total_items; item += units) {
        const Item w = decode_item<kBM>(ss, p, item);
        int b0, b1;
        weight_blocks<false, SWIGLU, true>(p, w, b0, b1);
        const int my_n = cta_tokens(w, 0);
        const uint8_t* wsf0 = p.w_sf + (size_t(w.g) * nbr + b0) * p.nkb;
        const uint8_t* wsf1 = p.w_sf + (size_t(w.g) * nbr + b1) * p.nkb;
        for (int kb = 0; kb < p.nkb; ++kb, ++it) {
            const int s = it % C::kStages;
            const uint32_t par = (it / C::kStages) & 1u;
            if (lane == 0) ok = mbar_wait(smem_u32(&ss->empty[s]), par ^ 1u, ss, p.dev_status);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            const uint8_t* asf = p.a_sf + size_t(kb) * p.max_rows + w.row0;
            uint32_t wd[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int m = lane + 32 * j;  // row m0 = lane, m1 = j
                const uint32_t b = m < my_n ? asf[m] : 127u;
                wd[j] = b * 0x01010101u;
            }
            uint8_t* ch = sf_area + s * C::kSfStage;
            *reinterpret_cast<uint4*>(ch + 16 * lane) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
            const uint32_t w0 = uint32_t(wsf0[kb]) * 0x01010101u;
            const uint32_t w1 = uint32_t(wsf1[kb]) * 0x01010101u;
            *reinterpret_cast<uint4*>(ch + 512 + 16 * lane) = make_uint4(w0, w0, w0, w0);
            *reinterpret_cast<uint4*>(ch + 1024 + 16 * lane) = make_uint4(w1, w1, w1, w1);
            // visible to the tensor core's copy (async proxy) before the signal
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&ss->sfull[s]));
        }
    }
    __syncwarp();
}

// warp 1, one thread
template <bool SWIGLU>
__device__ __forceinline__ void mx_mma_issuer(const GemmParams& p, uint8_t* smem, uint8_t* sf_area,
                                              SharedState* ss, uint32_t tmem_base, int unit,
                                              int units) {
    using C = MxCfg<SWIGLU>;
    const int lane = threadIdx.x & 31;
    const int total_items = ss->total_items;
    if (lane == 0) {
        uint32_t it = 0, n_item = 0;
        bool ok = true;
        for (int item = unit; ok && item < total_items; item += units, ++n_item) {
            // the epilogue has moved the previous item's accumulator out
            ok = mbar_wait(smem_u32(&ss->tempty[0]), (n_item & 1u) ^ 1u, ss, p.dev_status);
            if (!ok) break;
            tc_fence_after();
            for (int kb = 0; kb < p.nkb; ++kb, ++it) {
                const int s = it % C::kStages;
                const uint32_t par = (it / C::kStages) & 1u;
                ok = mbar_wait(smem_u32(&ss->full[s]), par, ss, p.dev_status) &&
                     mbar_wait(smem_u32(&ss->sfull[s]), par, ss, p.dev_status);
                if (!ok) break;
                tc_fence_after();
                const uint32_t ta = tmem_base + C::kSfCol + 12 * s, tb = ta + 4;
                const uint32_t ch = smem_u32(sf_area + s * C::kSfStage);
                tmem_cp_sf(ta, sf_desc(ch));
                tmem_cp_sf(tb, sf_desc(ch + 512));
                tmem_cp_sf(tb + 4, sf_desc(ch + 1024));
                const uint32_t st = smem_u32(smem + size_t(s) * C::kStageBytes);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_mx(tmem_base, sw128_desc(st + kk * 32), sw128_desc(st + kTileBytes + kk * 32),
                           idesc_mx(128, 256, uint32_t(kk)), (kb > 0 || kk > 0) ? 1u : 0u,
                           ta | (uint32_t(kk) << 30), tb | (uint32_t(kk) << 30));
                mma_commit<false>(smem_u32(&ss->empty[s]));
            }
            if (!ok) break;
            mma_commit<false>(smem_u32(&ss->tfull[0]));
        }
        mma_commit<false>(smem_u32(&ss->drain));
        mbar_quiesce(smem_u32(&ss->drain), 0, ss, nullptr);
    }
    __syncwarp();
}

// warps 4-11: thread (w, l) owns token row 32 (w % 4) + l and half h = (w-4)/4
// of the 256 columns (same mapping as the promotion form's epilogue).
template <bool SWIGLU>
__device__ __forceinline__ void mx_epilogue(const GemmParams& p, SharedState* ss, char* park_area,
                                            uint32_t tmem_base, const CUtensorMap* map_o, int unit,
                                            int units) {
    using C = MxCfg<SWIGLU>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int total_items = ss->total_items;
    const int q = warp & 3;
    const int half = (warp - 4) >> 2;
    const int r = q * 32 + lane;
    const uint32_t lane_addr = tmem_base + (uint32_t(q * 32) << 16);
    const int c0 = SWIGLU ? 64 * half : 128 * half;
    const int c1 = SWIGLU ? 128 + 64 * half : 128 * half + 64;
    char* const wpark = park_area + (warp - 4) * (C::kParkBoxes * kBoxBytes);
    uint32_t n_item = 0, parity = 0;
    bool ok = true;
    for (int item = unit; item < total_items; item += units, ++n_item, parity ^= 1u) {
        const Item w = decode_item<kBM>(ss, p, item);
        if (lane == 0) ok = mbar_wait(smem_u32(&ss->tfull[0]), n_item & 1u, ss, p.dev_status);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        const int my_n = cta_tokens(w, 0);
        const size_t row = size_t(w.row0) + r;
        if (!SWIGLU) {
            uint64_t acc2[64];
            if (ok) {
                __syncwarp();
                tc_fence_after();
                uint32_t v[64];
                tmem_ld64(lane_addr + c0, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) acc2[i] = pack2(v[2 * i], v[2 * i + 1]);
                tmem_ld64(lane_addr + c1, v);
#pragma unroll
                for (int i = 0; i < 32; ++i) acc2[32 + i] = pack2(v[2 * i], v[2 * i + 1]);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&ss->tempty[0]));  // accumulator free
            } else {
#pragma unroll
                for (int i = 0; i < 64; ++i) acc2[i] = 0;
            }
            store_rows<64, 1>(p, acc2, wpark, map_o, lane, my_n - q * 32, row, w.row0 + q * 32,
                              w.f * 256 + half * 128);
        } else {
            // gate (acc[0..63]) and up (acc[64..127]) of this thread's 64 features
            float acc[128];
            if (ok) {
                __syncwarp();
                tc_fence_after();
                uint32_t v[64];
                tmem_ld64(lane_addr + c0, v);
#pragma unroll
                for (int i = 0; i < 64; ++i) acc[i] = __uint_as_float(v[i]);
                tmem_ld64(lane_addr + c1, v);
#pragma unroll
                for (int i = 0; i < 64; ++i) acc[64 + i] = __uint_as_float(v[i]);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&ss->tempty[0]));  // accumulator free
            } else {
#pragma unroll
                for (int i = 0; i < 128; ++i) acc[i] = 0.0f;
            }
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                const float g = acc[i];
                const float hv = __fdividef(g, 1.0f + __expf(-g)) * acc[64 + i];
                acc[i] = hv;
                amax = fmaxf(amax, fabsf(hv));
            }
            ss->red[parity][half][r] = amax;
            named_bar(1, kPromoters * 32);
            amax = fmaxf(amax, ss->red[parity][half ^ 1][r]);
            const int e = pow2_exponent(amax);
            const float inv = pow2_inverse(e);
            if (r < my_n) {
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
                if (half == 0) p.out_sf[size_t(w.f) * p.max_rows + row] = uint8_t(e + 127);
            }
        }
        const bool any_abort = named_bar_or(
            2, kPromoters * 32, !ok || *reinterpret_cast<volatile int*>(&ss->abort_flag));
        if (any_abort) break;
    }
    if (!SWIGLU && lane == 0) bulk_wait_all();
    __syncwarp();
    tc_fence_before();
}

template <bool SWIGLU>
__global__ void __launch_bounds__(kThreads, 1)
    mx_gemm_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ AMaps maps_a,
                   const __grid_constant__ CUtensorMap map_o, const GemmParams p) {
    using C = MxCfg<SWIGLU>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    char* park = reinterpret_cast<char*>(smem + C::kRingBytes);
    uint8_t* sf_area = smem + C::kRingBytes + C::kParkBytes;
    SharedState* ss = reinterpret_cast<SharedState*>(sf_area + C::kSfBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int unit = int(blockIdx.x), units = int(gridDim.x);
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(smem_u32(&ss->full[s]), 1);
            mbar_init(smem_u32(&ss->empty[s]), 1);
            mbar_init(smem_u32(&ss->sfull[s]), 1);
        }
        mbar_init(smem_u32(&ss->tfull[0]), 1);
        mbar_init(smem_u32(&ss->tempty[0]), kPromoters);
        mbar_init(smem_u32(&ss->drain), 1);
        ss->wait_limit = p.wait_limit_ns;
        ss->abort_flag = 0;
        ss->peer_abort = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) tmem_alloc_all<false>(smem_u32(&ss->tmem_base));
    const int G = p.n_groups;
    int bad = 0;
    for (int i = threadIdx.x; i <= G; i += kThreads) {
        const int v = p.group_offsets[i];
        ss->goff[i] = v;
        if (v < 0 || v > p.max_rows || (i > 0 && v < p.group_offsets[i - 1])) bad = 1;
    }
    if (__syncthreads_or(bad)) {
        if (threadIdx.x == 0) set_status(p.dev_status, MOE_DEV_BAD_INPUT);
        for (int i = threadIdx.x; i <= G; i += kThreads) ss->goff[i] = 0;
        __syncthreads();
    }
    {
        constexpr int PER = (kMaxGroups + kThreads) / kThreads;
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
        if (warp == 0) mx_producer<SWIGLU>(p, &map_w, maps_a, smem, ss, unit, units);
        else if (warp == 1) mx_mma_issuer<SWIGLU>(p, smem, sf_area, ss, tmem_base, unit, units);
        else if (warp == 2) mx_scale_loader<SWIGLU>(p, sf_area, ss, unit, units);
    } else {
        set_max_regs_inc<208>();
        mx_epilogue<SWIGLU>(p, ss, park, tmem_base, &map_o, unit, units);
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_free_all<false>(tmem_base);
    }
}

template <bool SWIGLU>
int launch_mx(const GemmParams& p, const CUtensorMap& mw, const AMaps& ma, const CUtensorMap& mo,
              cudaStream_t st) {
    if (cudaFuncSetAttribute(mx_gemm_kernel<SWIGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(mx_smem_bytes<SWIGLU>())) != cudaSuccess)
        return MOE_ERR_CUDA;
    mx_gemm_kernel<SWIGLU><<<sm_count(), kThreads, mx_smem_bytes<SWIGLU>(), st>>>(mw, ma, mo, p);
    return check_launch();
}

// CTA pairs the device can hold at once for a pair kernel (cached per device).
template <bool SWIGLU>
int pair_units() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (cache[dev] == 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (sm_count() / 2), 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = smem_bytes<true, SWIGLU, true>();
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaFuncSetAttribute(grouped_gemm_kernel<true, SWIGLU, true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(smem_bytes<true, SWIGLU, true>())) != cudaSuccess ||
            cudaOccupancyMaxActiveClusters(&n, grouped_gemm_kernel<true, SWIGLU, true>, &cfg) !=
                cudaSuccess || n < 1) {
            (void)cudaGetLastError();
            n = -1;  // pairs unavailable on this device
        }
        cache[dev] = std::min(n, sm_count() / 2);
    }
    return cache[dev];
}

template <bool PAIR, bool SWIGLU, bool WIDE>
int launch(const GemmParams& p, const CUtensorMap& mw, const AMaps& ma, const CUtensorMap& mo,
           int units, cudaStream_t st) {
    if (cudaFuncSetAttribute(grouped_gemm_kernel<PAIR, SWIGLU, WIDE>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(smem_bytes<PAIR, SWIGLU, WIDE>())) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (!PAIR) {
        grouped_gemm_kernel<PAIR, SWIGLU, WIDE><<<sm_count(), kThreads, smem_bytes<PAIR, SWIGLU, WIDE>(), st>>>(
            mw, ma, mo, p);
        return check_launch();
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * units, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem_bytes<PAIR, SWIGLU, WIDE>();
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, grouped_gemm_kernel<PAIR, SWIGLU, WIDE>, mw, ma, mo, p) != cudaSuccess)
        return MOE_ERR_CUDA;
    return check_launch();
}

// ============================================== weight-gradient form (K-grouped)
// out[g] (fp32 [M, N]) = sum over the K blocks of group g of the products of
// A rows and B rows, with a scale per (row, K block) on BOTH operands: the
// weight gradients, whose contraction runs over one expert's token rows and
// whose two operands are activations quantised in 128x1 tiles along the
// tokens ("DeepSeek-V3 Technical Report" notes page, section "FP8 mixed
// precision training": all three linear GEMMs take FP8 inputs; the
// transposed activations need tiles along the other dimension).  A and B are
// stored transposed, K (the tokens, each group's rows padded to a multiple of
// 128) contiguous, so the tensor core sees ordinary K-major tiles; a group is
// a range of K blocks, not of rows.  The promotion is the forward's with the
// combined scale sa[row of A] * sb[row of B] per element (one more multiply
// per pair of values).  Every item covers 128 rows of A and 256 of B; an
// item whose group has no K blocks stores zeros (an expert no token chose).
struct WgCfg {
    static constexpr int kStages = 3;
    static constexpr int kStageBytes = kTileBytes + 256 * 128;  // A tile + two B boxes
    static constexpr int kRingBytes = kStages * kStageBytes;
    static constexpr int kParkBytes = kPromoters * kBoxBytes;
    static constexpr int kSbBytes = kScaleSlots * 256 * 4;      // B scales of a K block
    static constexpr int kBufs = 2;                             // 256-column TMEM partials
};
constexpr size_t wg_smem_bytes() {
    return size_t(WgCfg::kRingBytes) + WgCfg::kParkBytes + WgCfg::kSbBytes +
           sizeof(SharedState) + 1024;
}
static_assert(wg_smem_bytes() <= 232448, "dynamic shared memory above the sm_100 limit per CTA");

struct WgParams {
    const int32_t* kb_offsets;  // [n_groups + 1] K-block ranges of the groups
    int n_groups;
    int m, n;                   // rows of A and of B (output [n_groups, m, n])
    int nkb_total;              // K blocks of A and B
    int m_tiles, n_tiles;       // m / 128, n / 256
    const float* a_scales;      // [nkb_total, m]
    const float* b_scales;      // [nkb_total, n]
    int* dev_status;
    uint64_t wait_limit_ns;
    GemmParams out;             // epilogue fields (fp32 output, row pitch n)
};

struct WgItem {
    int g, mt, f, kb0, kb1;
};
__device__ __forceinline__ WgItem wg_item(const SharedState* ss, const WgParams& p, int item) {
    const int per = p.m_tiles * p.n_tiles;
    WgItem w;
    w.g = item / per;
    const int local = item - w.g * per;
    w.f = local / p.m_tiles;  // m tiles fastest: neighbouring CTAs share B
    w.mt = local - w.f * p.m_tiles;
    w.kb0 = ss->goff[w.g];
    w.kb1 = ss->goff[w.g + 1];
    return w;
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
                 : "memory");
}
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

__device__ __forceinline__ void wg_producer(const WgParams& p, const CUtensorMap* map_a,
                                            const CUtensorMap* map_b, uint8_t* smem,
                                            SharedState* ss, int unit, int units) {
    using C = WgCfg;
    const int lane = threadIdx.x & 31;
    const int total_items = ss->total_items;
    uint32_t it = 0, issued_mask = 0, issued_parity = 0;
    bool ok = true;
    for (int item = unit; ok && item < total_items; item += units) {
        const WgItem w = wg_item(ss, p, item);
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
            const int s = it % C::kStages;
            const uint32_t par = (it / C::kStages) & 1u;
            if (lane == 0) ok = mbar_wait(smem_u32(&ss->empty[s]), par ^ 1u, ss, p.dev_status);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            if (lane == 0) {
                uint8_t* st = smem + size_t(s) * C::kStageBytes;
                const uint32_t fb = smem_u32(&ss->full[s]);
                mbar_arrive_expect_tx(fb, uint32_t(C::kStageBytes));
                tma_load_2d<false>(smem_u32(st), map_a, fb, kb * 128, w.mt * 128);
                tma_load_2d<false>(smem_u32(st + kTileBytes), map_b, fb, kb * 128, w.f * 256);
                tma_load_2d<false>(smem_u32(st + 2 * kTileBytes), map_b, fb, kb * 128,
                                   w.f * 256 + 128);
                issued_mask |= 1u << s;
                issued_parity = (issued_parity & ~(1u << s)) | (par << s);
            }
        }
    }
    if (!ok && lane == 0)
        for (int s = 0; s < C::kStages; ++s)
            if ((issued_mask >> s) & 1u)
                mbar_quiesce(smem_u32(&ss->full[s]), (issued_parity >> s) & 1u, ss, nullptr);
    __syncwarp();
}

// warp 2: per K block, the 128 A scales into sa[slot] and the 256 B scales
// into the slot's row of sb_area (16-byte asynchronous copies).
__device__ __forceinline__ void wg_scale_loader(const WgParams& p, float* sb_area,
                                                SharedState* ss, int unit, int units) {
    const int lane = threadIdx.x & 31;
    const int total_items = ss->total_items;
    uint32_t cit = 0;
    bool ok = true;
    for (int item = unit; ok && item < total_items; item += units) {
        const WgItem w = wg_item(ss, p, item);
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++cit) {
            const int c = cit % kScaleSlots;
            if (lane == 0)
                ok = mbar_wait(smem_u32(&ss->sempty[c]), ((cit / kScaleSlots) & 1u) ^ 1u, ss,
                               p.dev_status);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            const float* sa = p.a_scales + size_t(kb) * p.m + w.mt * 128;
            const float* sb = p.b_scales + size_t(kb) * p.n + w.f * 256;
            cp_async16(&ss->sa[c][4 * lane], sa + 4 * lane);
            cp_async16(sb_area + c * 256 + 4 * lane, sb + 4 * lane);
            cp_async16(sb_area + c * 256 + 128 + 4 * lane, sb + 128 + 4 * lane);
            cp_async_arrive(smem_u32(&ss->sfull[c]));
        }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncwarp();
}

__device__ __forceinline__ void wg_mma_issuer(const WgParams& p, uint8_t* smem, SharedState* ss,
                                              uint32_t tmem_base, int unit, int units) {
    using C = WgCfg;
    const int lane = threadIdx.x & 31;
    const int total_items = ss->total_items;
    if (lane == 0) {
        uint32_t it = 0;
        bool ok = true;
        const uint32_t idesc = idesc_e4m3(128, 256);
        for (int item = unit; ok && item < total_items; item += units) {
            const WgItem w = wg_item(ss, p, item);
            for (int kb = w.kb0; ok && kb < w.kb1; ++kb, ++it) {
                const int s = it % C::kStages;
                const uint32_t buf = it % C::kBufs;
                ok = mbar_wait(smem_u32(&ss->full[s]), (it / C::kStages) & 1u, ss, p.dev_status) &&
                     mbar_wait(smem_u32(&ss->tempty[buf]), ((it / C::kBufs) & 1u) ^ 1u, ss,
                               p.dev_status);
                if (!ok) break;
                tc_fence_after();
                const uint32_t st = smem_u32(smem + size_t(s) * C::kStageBytes);
                const uint32_t d = tmem_base + buf * 256;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_e4m3<false>(d, sw128_desc(st + kk * 32),
                                    sw128_desc(st + kTileBytes + kk * 32), idesc, kk > 0 ? 1u : 0u);
                mma_commit<false>(smem_u32(&ss->empty[s]));  // stage free, partial ready
            }
        }
        mma_commit<false>(smem_u32(&ss->drain));
        mbar_quiesce(smem_u32(&ss->drain), 0, ss, nullptr);
    }
    __syncwarp();
}

// Two B-scale pairs from shared memory in one 16-byte load that the compiler
// keeps in program order (plain loads were all hoisted to the top of the K
// block, and the registers they took spilled the accumulators).
__device__ __forceinline__ void ld_shared_volatile2(const uint64_t* p, uint64_t& a, uint64_t& b) {
    asm volatile("ld.volatile.shared.v2.b64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "r"(smem_u32(p)));
}

// acc2[o + i] += v pair i * (sa * sb pair o + i) for 16 pairs, eight pairs
// of B scales at a time.
__device__ __forceinline__ void wg_fold(uint64_t (&acc2)[64], const uint32_t (&v)[32],
                                        uint64_t sa2, const uint64_t* sb2, int o) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        uint64_t s[8];
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
            uint64_t b0, b1;
            ld_shared_volatile2(sb2 + o + 8 * j + i, b0, b1);
            s[i] = fmul2(sa2, b0);
            s[i + 1] = fmul2(sa2, b1);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i)
            ffma2(acc2[o + 8 * j + i], pack2(v[2 * (8 * j + i)], v[2 * (8 * j + i) + 1]), s[i]);
    }
}

// warps 4-11: thread (w, l) owns A row 32 (w % 4) + l of the item and the
// 128 B rows [128 h, 128 h + 128) of its 256, h = (w - 4) / 4.
__device__ __forceinline__ void wg_promoter(const WgParams& p, SharedState* ss,
                                            const float* sb_area, char* park_area,
                                            uint32_t tmem_base, const CUtensorMap* map_o,
                                            int unit, int units) {
    using C = WgCfg;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int total_items = ss->total_items;
    const int q = warp & 3;
    const int half = (warp - 4) >> 2;
    const int r = q * 32 + lane;
    const uint32_t lane_addr = tmem_base + (uint32_t(q * 32) << 16);
    const int c0 = 128 * half;
    uint32_t it = 0;
    bool ok = true;
    char* const wpark = park_area + (warp - 4) * kBoxBytes;
    for (int item = unit; item < total_items; item += units) {
        const WgItem w = wg_item(ss, p, item);
        uint64_t acc2[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) acc2[i] = 0;
        for (int kb = w.kb0; ok && kb < w.kb1; ++kb, ++it) {
            const uint32_t buf = it % C::kBufs;
            const int c = it % kScaleSlots;
            if (lane == 0) {
                ok = mbar_wait(smem_u32(&ss->empty[it % C::kStages]), (it / C::kStages) & 1u, ss,
                               p.dev_status);
                if (ok) ok = mbar_wait(smem_u32(&ss->sfull[c]), (it / kScaleSlots) & 1u, ss,
                                       p.dev_status);
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            __syncwarp();
            tc_fence_after();
            const float sa = ss->sa[c][r];
            const uint64_t sa2 = pack2(__float_as_uint(sa), __float_as_uint(sa));
            const uint64_t* sb2 = reinterpret_cast<const uint64_t*>(sb_area + c * 256 + c0);
            const uint32_t tbase = lane_addr + buf * 256;
            // 32 columns per TMEM load (the per-column scales need the
            // registers a 64-column load would take)
            uint32_t v[32];
#pragma unroll
            for (int j = 0; j < 3; ++j) {
                tmem_ld32(tbase + c0 + 32 * j, v);
                wg_fold(acc2, v, sa2, sb2, 16 * j);
            }
            tmem_ld32(tbase + c0 + 96, v);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&ss->tempty[buf]));
            wg_fold(acc2, v, sa2, sb2, 48);
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&ss->sempty[c]));  // scales read
        }
        if (w.kb0 < w.kb1) {
            store_rows<64, 1>(p.out, acc2, wpark, map_o, lane, 32, 0,
                              w.g * p.m + w.mt * 128 + q * 32, w.f * 256 + c0);
        } else {
            // no K blocks (an expert no token chose): zeros, one 512-byte row
            // segment per store instruction, no staging
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out.out) +
                                                    size_t(w.g * p.m + w.mt * 128 + q * 32) * p.n +
                                                    w.f * 256 + c0) + lane;
#pragma unroll 4
            for (int i = 0; i < 32; ++i)
                dst[size_t(i) * (p.n / 4)] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        const bool any_abort = named_bar_or(
            2, kPromoters * 32, !ok || *reinterpret_cast<volatile int*>(&ss->abort_flag));
        if (any_abort) break;
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
    tc_fence_before();
}

__global__ void __launch_bounds__(kThreads, 1)
    wgrad_gemm_kernel(const __grid_constant__ CUtensorMap map_a,
                      const __grid_constant__ CUtensorMap map_b,
                      const __grid_constant__ CUtensorMap map_o, const WgParams p) {
    using C = WgCfg;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    char* park = reinterpret_cast<char*>(smem + C::kRingBytes);
    float* sb_area = reinterpret_cast<float*>(smem + C::kRingBytes + C::kParkBytes);
    SharedState* ss = reinterpret_cast<SharedState*>(smem + size_t(C::kRingBytes) + C::kParkBytes +
                                                     C::kSbBytes);
    const int warp = threadIdx.x >> 5;
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
        ss->wait_limit = p.wait_limit_ns;
        ss->abort_flag = 0;
        ss->peer_abort = 0u;
        ss->total_items = p.n_groups * p.m_tiles * p.n_tiles;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) tmem_alloc_all<false>(smem_u32(&ss->tmem_base));
    // K-block ranges (validated: non-decreasing, inside [0, nkb_total])
    const int G = p.n_groups;
    int bad = 0;
    for (int i = threadIdx.x; i <= G; i += kThreads) {
        const int v = p.kb_offsets[i];
        ss->goff[i] = v;
        if (v < 0 || v > p.nkb_total || (i > 0 && v < p.kb_offsets[i - 1])) bad = 1;
    }
    if (__syncthreads_or(bad)) {
        if (threadIdx.x == 0) set_status(p.dev_status, MOE_DEV_BAD_INPUT);
        for (int i = threadIdx.x; i <= G; i += kThreads) ss->goff[i] = 0;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = ss->tmem_base;
    const int unit = int(blockIdx.x), units = int(gridDim.x);
    if (warp < 4) {
        set_max_regs_dec<72>();
        if (warp == 0) wg_producer(p, &map_a, &map_b, smem, ss, unit, units);
        else if (warp == 1) wg_mma_issuer(p, smem, ss, tmem_base, unit, units);
        else if (warp == 2) wg_scale_loader(p, sb_area, ss, unit, units);
    } else {
        set_max_regs_inc<208>();
        wg_promoter(p, ss, sb_area, park, tmem_base, &map_o, unit, units);
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_free_all<false>(tmem_base);
    }
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

// Kernel form of a call: the number of CTA pairs to launch, or 0 for single
// CTAs.  CTA pairs halve the operand traffic per SM, but on B200 that
// traffic does not bound this kernel (the hand-off between the MMA and the
// promotion warps does, once per K block of 128 x 256 partials in both
// forms): measured, pairs and 256-column single CTAs run the 4096-row bf16
// GEMM at the same 1430 TFLOP/s and the skewed W2 within 1%, while pairs
// are 1.5x slower on the 257-expert prefill W13 (half of a pair's 256
// tokens are padding there).  Single CTAs are therefore the default;
// MOEFP8_GEMM_PAIR=1 in the environment selects pairs where the output
// width is a multiple of 256 (SwiGLU always is).
int gemm_pair_units(int n_groups, int max_rows, int n, bool swiglu) {
    (void)n_groups;
    (void)max_rows;
    const char* env = getenv("MOEFP8_GEMM_PAIR");
    const bool want = env && env[0] == '1' && (swiglu || n % 256 == 0);
    if (!want) return 0;
    return std::max(0, swiglu ? pair_units<true>() : pair_units<false>());
}

}  // namespace moe

using namespace moe;

extern "C" MOE_API int moe_grouped_gemm_form(int n_groups, int max_rows, int n, int epilogue) {
    if (n_groups < 1 || max_rows < 0 || n <= 0 || n % 128) return 0;
    if (epilogue != MOE_EPI_F32 && epilogue != MOE_EPI_BF16 && epilogue != MOE_EPI_SWIGLU_QUANT)
        return 0;
    if (epilogue == MOE_EPI_SWIGLU_QUANT && n % 256) return 0;
    return gemm_pair_units(n_groups, max_rows, n, epilogue == MOE_EPI_SWIGLU_QUANT) > 0 ? 2 : 1;
}

namespace moe {
int grouped_gemm_fp8(int n_groups, const int32_t* group_offsets, int max_rows, const uint8_t* a,
                     const float* a_scales, int k, const uint8_t* w, const float* w_scales, int n,
                     int epilogue, void* out, float* out_scales, const int32_t* group_weight,
                     int n_weights, int* dev_status, void* stream);
}

extern "C" MOE_API int moe_grouped_gemm_fp8(int n_groups, const int32_t* group_offsets,
                                            int max_rows, const uint8_t* a,
                                            const float* a_scales, int k, const uint8_t* w,
                                            const float* w_scales, int n, int epilogue,
                                            void* out, float* out_scales, int* dev_status,
                                            void* stream) {
    return grouped_gemm_fp8(n_groups, group_offsets, max_rows, a, a_scales, k, w, w_scales, n,
                            epilogue, out, out_scales, nullptr, n_groups, dev_status, stream);
}

extern "C" MOE_API int moe_grouped_gemm_fp8_indexed(
    int n_groups, const int32_t* group_offsets, const int32_t* group_weight, int n_weights,
    int max_rows, const uint8_t* a, const float* a_scales, int k, const uint8_t* w,
    const float* w_scales, int n, int epilogue, void* out, float* out_scales, int* dev_status,
    void* stream) {
    if (!group_weight) return MOE_ERR_NULL;
    if (n_weights < 1) return MOE_ERR_SHAPE;
    return grouped_gemm_fp8(n_groups, group_offsets, max_rows, a, a_scales, k, w, w_scales, n,
                            epilogue, out, out_scales, group_weight, n_weights, dev_status, stream);
}

int moe::grouped_gemm_fp8(int n_groups, const int32_t* group_offsets, int max_rows,
                          const uint8_t* a, const float* a_scales, int k, const uint8_t* w,
                          const float* w_scales, int n, int epilogue, void* out,
                          float* out_scales, const int32_t* group_weight, int n_weights,
                          int* dev_status, void* stream) {
    if (n_groups < 1 || n_groups > kMaxGroups || max_rows < 0 || k <= 0 || k % 128 || n <= 0 ||
        n % 128)
        return MOE_ERR_SHAPE;
    if (epilogue != MOE_EPI_F32 && epilogue != MOE_EPI_BF16 && epilogue != MOE_EPI_SWIGLU_QUANT)
        return MOE_ERR_ARG;
    if (epilogue == MOE_EPI_SWIGLU_QUANT && n % 256) return MOE_ERR_SHAPE;
    if (!group_offsets || !w || !w_scales) return MOE_ERR_NULL;
    if (max_rows == 0) return MOE_OK;  // no rows: nothing read or written
    if (!out || (epilogue == MOE_EPI_SWIGLU_QUANT && !out_scales)) return MOE_ERR_NULL;
    if (!a || !a_scales) return MOE_ERR_NULL;
    if (!aligned16(a) || !aligned16(w) || !aligned16(out)) return MOE_ERR_ALIGN;
    if (int64_t(n_weights) * n > INT32_MAX) return MOE_ERR_SHAPE;
    if (!device_is_sm100()) return MOE_ERR_DEVICE;

    const bool swiglu = epilogue == MOE_EPI_SWIGLU_QUANT;
    const int units = gemm_pair_units(n_groups, max_rows, n, swiglu);
    const bool pair = units > 0;

    GemmParams p;
    p.group_offsets = group_offsets;
    p.n_groups = n_groups;
    p.max_rows = max_rows;
    p.a_scales = a_scales;
    p.k = k;
    p.nkb = k / 128;
    p.w_scales = w_scales;
    p.n = n;
    // 256 output columns per tile wherever n allows (a TMEM round trip per K
    // block then carries twice the work); 128 otherwise
    const bool wide = pair || swiglu || n % 256 == 0;
    p.n_ftiles = wide ? n / 256 : n / 128;
    p.epilogue = epilogue;
    p.out = out;
    p.out_scales = out_scales;
    p.dev_status = dev_status;
    p.wait_limit_ns = wait_limit_ns();
    p.fault = fault_injection();
    p.group_weight = group_weight;
    p.n_weights = n_weights;

    CUtensorMap mw, mo;
    AMaps ma;
    if (!make_map(&mw, w, uint64_t(n_weights) * n, uint64_t(k), 128)) return MOE_ERR_CUDA;
    for (int i = 0; i < kABoxes; ++i)
        if (!make_map(&ma.m[i], a, uint64_t(max_rows), uint64_t(k), uint32_t(128 >> i)))
            return MOE_ERR_CUDA;
    if (swiglu) mo = mw;  // unused by the SwiGLU epilogue
    else if (!make_out_map(&mo, out, uint64_t(max_rows), uint64_t(n), epilogue == MOE_EPI_BF16))
        return MOE_ERR_CUDA;
    cudaStream_t st = as_stream(stream);
    if (pair)
        return swiglu ? launch<true, true, true>(p, mw, ma, mo, units, st)
                      : launch<true, false, true>(p, mw, ma, mo, units, st);
    if (swiglu) return launch<false, true, true>(p, mw, ma, mo, 0, st);
    return wide ? launch<false, false, true>(p, mw, ma, mo, 0, st)
                : launch<false, false, false>(p, mw, ma, mo, 0, st);
}

extern "C" MOE_API int moe_grouped_gemm_mxfp8(int n_groups, const int32_t* group_offsets,
                                              int max_rows, const uint8_t* a, const uint8_t* a_sf,
                                              int k, const uint8_t* w, const uint8_t* w_sf, int n,
                                              int epilogue, void* out, uint8_t* out_sf,
                                              int* dev_status, void* stream) {
    if (n_groups < 1 || n_groups > kMaxGroups || max_rows < 0 || k <= 0 || k % 128 || n <= 0 ||
        n % 256)
        return MOE_ERR_SHAPE;
    if (epilogue != MOE_EPI_F32 && epilogue != MOE_EPI_BF16 && epilogue != MOE_EPI_SWIGLU_QUANT)
        return MOE_ERR_ARG;
    if (!group_offsets || !w || !w_sf) return MOE_ERR_NULL;
    if (max_rows == 0) return MOE_OK;  // no rows: nothing read or written
    if (!out || (epilogue == MOE_EPI_SWIGLU_QUANT && !out_sf)) return MOE_ERR_NULL;
    if (!a || !a_sf) return MOE_ERR_NULL;
    if (!aligned16(a) || !aligned16(w) || !aligned16(out)) return MOE_ERR_ALIGN;
    if (int64_t(n_groups) * n > INT32_MAX) return MOE_ERR_SHAPE;
    if (!device_is_sm100()) return MOE_ERR_DEVICE;
    const bool swiglu = epilogue == MOE_EPI_SWIGLU_QUANT;
    GemmParams p = {};
    p.group_offsets = group_offsets;
    p.n_groups = n_groups;
    p.max_rows = max_rows;
    p.k = k;
    p.nkb = k / 128;
    p.n = n;
    p.n_ftiles = n / 256;
    p.epilogue = epilogue;
    p.out = out;
    p.dev_status = dev_status;
    p.wait_limit_ns = wait_limit_ns();
    p.fault = kFaultNone;
    p.a_sf = a_sf;
    p.w_sf = w_sf;
    p.out_sf = out_sf;
    p.group_weight = nullptr;
    p.n_weights = n_groups;
    CUtensorMap mw, mo;
    AMaps ma;
    if (!make_map(&mw, w, uint64_t(n_groups) * n, uint64_t(k), 128)) return MOE_ERR_CUDA;
    for (int i = 0; i < kABoxes; ++i)
        if (!make_map(&ma.m[i], a, uint64_t(max_rows), uint64_t(k), uint32_t(128 >> i)))
            return MOE_ERR_CUDA;
    if (swiglu) mo = mw;  // unused by the SwiGLU epilogue
    else if (!make_out_map(&mo, out, uint64_t(max_rows), uint64_t(n), epilogue == MOE_EPI_BF16))
        return MOE_ERR_CUDA;
    cudaStream_t st = as_stream(stream);
    return swiglu ? launch_mx<true>(p, mw, ma, mo, st) : launch_mx<false>(p, mw, ma, mo, st);
}

extern "C" MOE_API int moe_grouped_gemm_wgrad(int n_groups, const int32_t* kb_offsets,
                                              int nkb_total, const uint8_t* a_t,
                                              const float* a_scales, int m, const uint8_t* b_t,
                                              const float* b_scales, int n, float* out,
                                              int* dev_status, void* stream) {
    if (n_groups < 1 || n_groups > kMaxGroups || nkb_total < 0 || m <= 0 || m % 128 || n <= 0 ||
        n % 256)
        return MOE_ERR_SHAPE;
    if (int64_t(n_groups) * m > INT32_MAX || int64_t(nkb_total) * 128 > INT32_MAX)
        return MOE_ERR_SHAPE;
    if (!kb_offsets || !out) return MOE_ERR_NULL;
    const bool empty_k = nkb_total == 0;
    if (!empty_k && (!a_t || !a_scales || !b_t || !b_scales)) return MOE_ERR_NULL;
    if (!aligned16(out) || (!empty_k && (!aligned16(a_t) || !aligned16(b_t) ||
                                         !aligned16(a_scales) || !aligned16(b_scales))))
        return MOE_ERR_ALIGN;
    if (!device_is_sm100()) return MOE_ERR_DEVICE;
    cudaStream_t st = as_stream(stream);
    if (empty_k) {
        // no token rows at all: every gradient is zero
        return cudaMemsetAsync(out, 0, sizeof(float) * size_t(n_groups) * m * n, st) ==
                       cudaSuccess
                   ? MOE_OK
                   : MOE_ERR_CUDA;
    }
    WgParams p;
    p.kb_offsets = kb_offsets;
    p.n_groups = n_groups;
    p.m = m;
    p.n = n;
    p.nkb_total = nkb_total;
    p.m_tiles = m / 128;
    p.n_tiles = n / 256;
    p.a_scales = a_scales;
    p.b_scales = b_scales;
    p.dev_status = dev_status;
    p.wait_limit_ns = wait_limit_ns();
    p.out = GemmParams{};
    p.out.epilogue = MOE_EPI_F32;
    p.out.out = out;
    p.out.n = n;
    p.out.dev_status = dev_status;
    CUtensorMap ma, mb, mo;
    const uint64_t kcols = uint64_t(nkb_total) * 128;
    if (!make_map(&ma, a_t, uint64_t(m), kcols, 128) || !make_map(&mb, b_t, uint64_t(n), kcols, 128) ||
        !make_out_map(&mo, out, uint64_t(n_groups) * m, uint64_t(n), false))
        return MOE_ERR_CUDA;
    if (cudaFuncSetAttribute(wgrad_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(wg_smem_bytes())) != cudaSuccess)
        return MOE_ERR_CUDA;
    wgrad_gemm_kernel<<<sm_count(), kThreads, wg_smem_bytes(), st>>>(ma, mb, mo, p);
    return check_launch();
}
