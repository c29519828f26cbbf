// Token-to-expert routing ("DeepSeek-V3 Technical Report" notes page,
// section "DeepSeekMoE and auxiliary-loss-free load balancing"): sigmoid
// affinity, bias for the routing decision only, group-limited top-K (the
// "at most M nodes" rule with expert groups standing in for nodes), gates
// normalised from the unbiased affinities, and the per-batch expert load
// histogram.  Gating stays in high precision (section "FP8 mixed precision
// training"): a logit is the FP64 dot product summed in ascending k, rounded
// to fp32, so the result is reproducible bit for bit.
//
// Computing all T*N_r logits that way is FP64-bound.  The path here gets
// them from exact integer arithmetic on the tensor cores, decides the
// routing from the result wherever a rigorous bound allows, and evaluates
// the defining FP64 sum only where it is still needed:
//   1. route_slice_kernel: every row v (of x and of E) is written as
//      v = 2^(sigma-28) * (X0*2^21 + X1*2^14 + X2*2^7 + X3) + r with signed
//      7-bit digits X0..X3 (int8 planes), sigma the exponent of max |v|;
//      r = 0 unless the row has values below 2^(sigma-21) of its maximum.
//      Also ||v||_1, ||v||_2 and the exactness of the row;
//   2. route_imma_kernel: tcgen05.mma kind::i8 over the digit planes, the
//      16 plane products summed per level L = s + r into seven exact int32
//      TMEM accumulators; sum_k X_k E_k = sum_L 2^(7(6-L)) acc_L;
//   3. route_certify_kernel (warp per token): u~ from the levels (exact up to
//      one FP64 rounding when both rows are exact); a bound B on the distance
//      to the defining FP64 sum (the rows' remainders, gamma_d(FP64) *
//      ||x|| ||E||, the FP64 roundings); intervals for every biased score s'
//      (sigmoid is 1/4-Lipschitz; fp32 roundings are bounded); the group /
//      top-K choice on the interval centres and a check that every chosen
//      interval lies strictly above every rejected one.  Certified tokens get
//      their chosen logits as fp32(u~) when [u~-B, u~+B] holds no fp32
//      rounding boundary; others go on a list;
//   4. the defining FP64 sum for the chosen logits that were not settled
//      in 3 and, when the list is short, for all N_r logits of every listed
//      token: route_exact_pairs_kernel (a warp per chosen logit) settles
//      those whose sum provably cannot round, from an exact parallel sum;
//      route_exact_chain_kernel (a warp per sum, operands streamed while one
//      lane adds in order) evaluates the rest in ascending k;
//      route_list_rows_kernel (a thread per sum) the listed tokens' rows
//      while the list is short, route_logits_list_kernel (64x64 FP64
//      tiles) when it is long;
//   5. route_select_kernel (warp per token): exact s and s' of the chosen
//      experts, slot order, gates and histogram for certified tokens; the
//      full selection on the exact logits for listed ones.
#include <float.h>
#include <math.h>

#include "tc.cuh"

namespace moe {
namespace {

// --------------------------------------------------------------- helpers
// Index checks of the routing kernels: an out-of-range index is skipped and
// reported (dev_status = MOE_DEV_BAD_INPUT; check[2*site] = 1 and
// check[2*site+1] = the offending value).  Sites: 0 list overflow, 1 list
// length, 2 pair index, 3 listed token, 4 chosen expert (certified path),
// 5 chosen expert (full path).
constexpr int kCheckWords = 16;

__device__ __forceinline__ void route_bad(int* dev_status, int32_t* check, int site, int value) {
    set_status(dev_status, MOE_DEV_BAD_INPUT);
    if (atomicCAS(&check[2 * site], 0, 1) == 0) check[2 * site + 1] = value;
}

// bf16 word pair -> doubles (exact)
__device__ __forceinline__ double bf16_lo_d(uint32_t w) { return (double)bf16_lo(w); }
__device__ __forceinline__ double bf16_hi_d(uint32_t w) { return (double)bf16_hi(w); }

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

__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// ------------------------------------------------------ 1. digit planes
// One warp per row; rows [0, T) are tokens (planes xp), [T, T+N) router rows
// (planes ep).  Plane s of a row set holds digit X_s of every value, planes
// stacked as [4][rows][d] int8.  Per row r:
//   rsc[r] = 2^(sigma-28), the unit of the integer X;
//   rex[r] = 1 when every value is exactly 2^(sigma-28) * X, 0 when some
//            value has bits below that unit, -1 when the row holds a
//            non-finite value;
//   r1[r] = sum |v - 2^(sigma-28) X| (the truncated remainders), l2[r] =
//            ||v||_2 (FP64, raised by 1 + nmargin to cover their rounding);
//   vmax[r], vmin[r] = max |v| (+inf for a non-finite row) and min |v| over
//            v != 0 (FLT_MAX for an all-zero row);
//   lb[r]  = the lowest bit any value of the row can carry: a bf16 value
//            in [2^e, 2^(e+1)) has no bit below 2^(e-7) (2^-133 below 2^-126).
// Block 0 also clears the two list counters and the check words of this call.
// With `staged`, the first pass keeps the row in the warp's slice of shared
// memory (d * 2 bytes; the launch provides kSliceWarps of them) and the
// second reads it from there; otherwise the second pass reads the row again.
constexpr int kSliceWarps = 4;
constexpr int kSliceStageMax = 32 * 1024;  // largest row staged per warp (d <= 16384)
__global__ void __launch_bounds__(kSliceWarps * 32) route_slice_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ E, int T, int N, int d,
    double nmargin, int staged, int8_t* __restrict__ xp, int8_t* __restrict__ ep,
    double* __restrict__ rsc, int32_t* __restrict__ rex, double* __restrict__ r1,
    double* __restrict__ l2, float* __restrict__ vmax, float* __restrict__ vmin,
    double* __restrict__ lb, int32_t* __restrict__ list_count, int32_t* __restrict__ pair_count,
    int32_t* __restrict__ check) {
    extern __shared__ __align__(16) uint4 slice_rows[];
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        *list_count = 0;
        *pair_count = 0;
    }
    if (blockIdx.x == 0 && threadIdx.x < kCheckWords) check[threadIdx.x] = 0;
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * kSliceWarps;
    uint4* const mine = slice_rows + (staged ? (threadIdx.x >> 5) * (d / 8) : 0);
    for (int r = blockIdx.x * kSliceWarps + (threadIdx.x >> 5); r < T + N; r += warps) {
        const bool is_x = r < T;
        const int rr = is_x ? r : r - T;
        const int nrows = is_x ? T : N;
        const uint4* row = reinterpret_cast<const uint4*>((is_x ? x : E) + int64_t(rr) * d);
        int8_t* planes = is_x ? xp : ep;
        float mx = 0.0f, mn = FLT_MAX;
        bool finite = true;
        __syncwarp();  // the previous row's second pass is done with the slice
#pragma unroll 4
        for (int v = lane; v < d / 8; v += 32) {
            const uint4 w = __ldg(row + v);
            if (staged) mine[v] = w;
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float a = fabsf(bf16_lo(ws[q])), b = fabsf(bf16_hi(ws[q]));
                finite = finite && a <= FLT_MAX && b <= FLT_MAX;
                mx = fmaxf(mx, fmaxf(a, b));
                if (a > 0.0f) mn = fminf(mn, a);
                if (b > 0.0f) mn = fminf(mn, b);
            }
        }
        mx = warp_max(mx);
        mn = warp_min(mn);
        finite = __all_sync(0xffffffffu, finite);  // (also orders the slice's stores)
        int sigma = 0;
        if (finite && mx > 0.0f) frexpf(mx, &sigma);  // mx < 2^sigma
        const double unit_inv = ldexp(1.0, 28 - sigma);
        bool exact = finite;
        double s1 = 0.0, s2 = 0.0;
        for (int v = lane; v < d / 8; v += 32) {
            const uint4 w = staged ? mine[v] : __ldg(row + v);
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
            // digit s of X is sign(X) * ((|X| >> 7(3-s)) & 127) (the truncating
            // base-128 digits: all share X's sign); four values' digits are
            // packed as magnitudes, then the negative ones negated bytewise
            uint32_t dg[4][2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t mag[4] = {0u, 0u, 0u, 0u}, neg = 0u;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int q = 4 * h + j;
                    const float f = (q & 1) ? bf16_hi(ws[q >> 1]) : bf16_lo(ws[q >> 1]);
                    s2 = fma((double)f, (double)f, s2);
                    const double xd = finite ? (double)f * unit_inv : 0.0;
                    const int X = __double2int_rz(xd);  // |X| < 2^28
                    exact = exact && (double)X == xd;
                    s1 += fabs(xd - (double)X);  // exact: a remainder below one unit
                    const uint32_t a = uint32_t(abs(X));
                    if (X < 0) neg |= 0xFFu << (8 * j);
                    mag[0] |= (a >> 21) << (8 * j);
                    mag[1] |= ((a >> 14) & 0x7Fu) << (8 * j);
                    mag[2] |= ((a >> 7) & 0x7Fu) << (8 * j);
                    mag[3] |= (a & 0x7Fu) << (8 * j);
                }
#pragma unroll
                for (int s = 0; s < 4; ++s) dg[s][h] = __vsub4(mag[s] ^ neg, neg);
            }
#pragma unroll
            for (int s = 0; s < 4; ++s)
                reinterpret_cast<uint2*>(planes + (int64_t(s) * nrows + rr) * d)[v] =
                    make_uint2(dg[s][0], dg[s][1]);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            s1 += __shfl_xor_sync(0xffffffffu, s1, o);
            s2 += __shfl_xor_sync(0xffffffffu, s2, o);
        }
        exact = __all_sync(0xffffffffu, exact);
        if (lane == 0) {
            vmax[r] = finite ? mx : INFINITY;
            vmin[r] = mn;
            int emin = 0;
            frexpf(mn < FLT_MAX ? mn : 1.0f, &emin);  // mn in [2^(emin-1), 2^emin)
            lb[r] = ldexp(1.0, max(emin - 1, -126) - 7);
            rsc[r] = ldexp(1.0, sigma - 28);
            rex[r] = finite ? (exact ? 1 : 0) : -1;
            r1[r] = ldexp(s1, sigma - 28) * (1.0 + nmargin);
            l2[r] = sqrt(s2) * (1.0 + nmargin);
        }
    }
}

// --------------------------------------------------- 2. integer logits
// One CTA per (128 tokens, 64 experts, K range): the four digit planes of
// both operands are streamed by TMA in 128-k stages (two stages in flight);
// one thread issues 16 plane products x 4 MMAs (M=128, N=64, K=32) per
// stage into seven TMEM accumulators (level L = s + r at columns 64L), and
// the four warps move the levels out: stored, or added atomically when K is
// split (integer addition: exact in any order).  Rows past T or N read other
// rows' digits or zeros and are never stored.
constexpr int kIM = 128, kIN = 64, kIK = 128, kIStages = 2, kLevels = 7;
constexpr int kIPlaneA = kIM * kIK, kIPlaneB = kIN * kIK;   // bytes per plane tile
constexpr int kIStageBytes = 4 * kIPlaneA + 4 * kIPlaneB;   // 96 KB

struct ImmaShared {
    uint64_t full[kIStages];
    uint64_t empty[kIStages];
    uint64_t done;
    uint32_t tmem_base;
    int abort;
};

constexpr size_t kImmaSmem = size_t(kIStages) * kIStageBytes + 1024 + sizeof(ImmaShared) + 64;

__global__ void __launch_bounds__(128, 1) route_imma_kernel(
    const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_e, int T,
    int N, int nchunks, int chunks_per_split, int32_t* __restrict__ acc, int* dev_status,
    uint64_t wait_ns) {
    extern __shared__ __align__(1024) uint8_t imma_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(imma_raw) + 1023) &
                                               ~uintptr_t(1023));
    ImmaShared* ss = reinterpret_cast<ImmaShared*>(smem + size_t(kIStages) * kIStageBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = blockIdx.x * kIM, e0 = blockIdx.y * kIN;
    const int c0 = blockIdx.z * chunks_per_split;
    const int c1 = min(nchunks, c0 + chunks_per_split);
    if (c0 >= c1) return;  // uniform over the CTA
    if (threadIdx.x == 0) {
        for (int i = 0; i < kIStages; ++i) {
            tc::mbar_init(tc::smem_u32(&ss->full[i]), 1);
            tc::mbar_init(tc::smem_u32(&ss->empty[i]), 1);
        }
        tc::mbar_init(tc::smem_u32(&ss->done), 1);
        ss->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                         tc::smem_u32(&ss->tmem_base))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = ss->tmem_base;
    if (warp == 0 && lane == 0) {
        // producer
        int issued = 0;
        for (int c = c0; c < c1; ++c, ++issued) {
            const int st = issued % kIStages;
            if (issued >= kIStages &&
                !tc::mbar_wait(tc::smem_u32(&ss->empty[st]), ((issued / kIStages) - 1) & 1,
                               &ss->abort, dev_status, wait_ns))
                break;
            const uint32_t bar = tc::smem_u32(&ss->full[st]);
            tc::mbar_arrive_expect_tx(bar, kIStageBytes);
            uint8_t* stage = smem + size_t(st) * kIStageBytes;
            for (int s = 0; s < 4; ++s)
                tc::tma_load_2d(tc::smem_u32(stage + s * kIPlaneA), &map_x, bar, c * kIK,
                                s * T + t0);
            for (int r = 0; r < 4; ++r)
                tc::tma_load_2d(tc::smem_u32(stage + 4 * kIPlaneA + r * kIPlaneB), &map_e, bar,
                                c * kIK, r * N + e0);
        }
        // the copies of the last stages have landed before the CTA moves on
        // (also after an abort: they write this CTA's shared memory)
        for (int i = max(0, issued - kIStages); i < issued; ++i)
            tc::mbar_quiesce(tc::smem_u32(&ss->full[i % kIStages]), (i / kIStages) & 1,
                             dev_status, wait_ns);
    } else if (warp == 1 && lane == 0) {
        // MMA issuer
        const uint32_t idesc = tc::idesc_s8(kIM, kIN);
        for (int c = c0, i = 0; c < c1; ++c, ++i) {
            const int st = i % kIStages;
            if (!tc::mbar_wait(tc::smem_u32(&ss->full[st]), (i / kIStages) & 1, &ss->abort,
                               dev_status, wait_ns))
                break;
            tc::fence_after();
            const uint32_t a0 = tc::smem_u32(smem + size_t(st) * kIStageBytes);
            const uint32_t b0 = a0 + 4 * kIPlaneA;
            for (int s = 0; s < 4; ++s)
                for (int r = 0; r < 4; ++r) {
                    const int L = s + r;
                    const bool first_of_level = (s == (L > 3 ? L - 3 : 0));
#pragma unroll
                    for (int kk = 0; kk < kIK / 32; ++kk) {
                        const uint32_t accumulate = (i == 0 && kk == 0 && first_of_level) ? 0u : 1u;
                        tc::mma_s8(tmem + uint32_t(L * kIN),
                                   tc::sw128_desc(a0 + s * kIPlaneA + kk * 32),
                                   tc::sw128_desc(b0 + r * kIPlaneB + kk * 32), idesc, accumulate);
                    }
                }
            tc::commit(tc::smem_u32(&ss->empty[st]));
        }
        tc::commit(tc::smem_u32(&ss->done));  // after every MMA issued above
    }
    __syncwarp();
    // levels out: warp w holds TMEM lanes (tokens) 32w .. 32w+31.  Every MMA
    // issued has completed once `done` fires, abort or not (TMEM is freed
    // below).
    bool ok = tc::mbar_quiesce(tc::smem_u32(&ss->done), 0, dev_status, wait_ns) &&
              !*reinterpret_cast<volatile int*>(&ss->abort);
    ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
    tc::fence_after();
    if (ok) {
        const int t = t0 + warp * 32 + lane;
        const bool split = gridDim.z > 1;
        for (int L = 0; L < kLevels; ++L) {
#pragma unroll
            for (int c = 0; c < kIN; c += 16) {
                uint32_t v[16];
                tc::tmem_ld16(tmem + (uint32_t(warp * 32) << 16) + uint32_t(L * kIN + c), v);
                if (t < T) {
                    int32_t* dst = acc + (int64_t(L) * T + t) * N + e0 + c;
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        if (e0 + c + j >= N) break;
                        if (split) atomicAdd(dst + j, int32_t(v[j]));
                        else dst[j] = int32_t(v[j]);
                    }
                }
            }
        }
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem)
                     : "memory");
    }
}

// ---------------------------------------------------------- 3. certify
// One warp per token.  u~ = 2^(sigma_t + sigma_i - 56) * sum_L 2^(7(6-L)) acc_L
// is the exact sum of the rows' integer parts up to one FP64 rounding;
//   B = r1(x_t) max|E_i| + r1(E_i) max|x_t| + gamma_d(FP64) ||x_t||_2 ||E_i||_2
//       + 2^-52 |u~| + tiny
// bounds |u~ - u_def| before u_def's fp32 rounding (the slicing remainders:
// sum |r_k E_k| + sum |X_k rho_k| with r1 the remainder sums; the error of
// the defining FP64 sum; the roundings of u~ and of u~ +- B).  The biased score s'_i of the definition lies within delta_i of
// centre_i = sigma(u~ + off_i) + b_i, where
//   delta_i = B'/4 + 2^-23 + 2^-24 |b_i| + 1e-14,
//   B' = B + 2^-23 (|u~| + |off_i| + B)
// (B' adds the fp32 roundings of u and of u + off; sigma is 1/4-Lipschitz;
// 2^-23 + 2^-24 |b_i| covers the fp32 roundings of s and s + b; 1e-14 the
// FP64 evaluation of sigma).  The interval ends are stored rounded outwards
// to fp32.  Groups and experts are chosen on the centres; the choice is
// certified when the lowest chosen lower end is strictly above the highest
// rejected upper end, for the groups and then for the experts inside the
// chosen groups.  A certified token's chosen logit is the exact fp32
// rounding of the level sum when both rows are sliced exactly and the
// defining sum provably does not round (sum_is_exact), else fp32(u~) when
// u~ - B and u~ + B round to the same fp32 value; otherwise (t, slot) goes
// on the pair list, to be summed.
constexpr int kCertWarps = 8;
__host__ __device__ constexpr int cert_pitch(int n) { return n + n / 32 + 1; }
__device__ __forceinline__ int cert_at(int i) { return i + (i >> 5); }

// sum_L 2^(7(6-L)) acc_L = hi * 2^28 + lo, both parts exact in int64.
__device__ __forceinline__ void level_parts(const int32_t* __restrict__ acc, int64_t plane,
                                            int64_t at, int64_t& hi, int64_t& lo) {
    hi = int64_t(acc[at]) * (1 << 14) + int64_t(acc[plane + at]) * (1 << 7) +
         int64_t(acc[2 * plane + at]);
    lo = int64_t(acc[3 * plane + at]) * (1 << 21) + int64_t(acc[4 * plane + at]) * (1 << 14) +
         int64_t(acc[5 * plane + at]) * (1 << 7) + int64_t(acc[6 * plane + at]);
}

__device__ __forceinline__ double level_sum(const int32_t* __restrict__ acc, int64_t plane,
                                            int64_t at) {
    int64_t hi, lo;
    level_parts(acc, plane, at, hi, lo);
    return (double)hi * 0x1p28 + (double)lo;
}

// Every product x_k E_k is a multiple of Q = lb(x_t) lb(E_i) and every
// partial sum of the defining FP64 sum is at most ||x_t||_2 ||E_i||_2 in
// magnitude; below 2^53 Q each partial sum is a double, so no addition
// rounds and the defining sum equals the exact sum, in any order.
__device__ __forceinline__ bool sum_is_exact(int t, int i, int T, const double* __restrict__ l2,
                                             const double* __restrict__ lb) {
    return l2[t] * l2[T + i] < 0x1p53 * (lb[t] * lb[T + i]);
}

// fp32(round-to-nearest-even) of (hi * 2^28 + lo) * scale, exactly: the sum
// is split into s = fl(hi*2^28 + lo) and its exact error e (TwoSum); s + e
// rounds like s unless s is the midpoint of two fp32 values, where e (if
// not zero) decides.  scale is a power of two.
__device__ __forceinline__ float exact_level_fp32(int64_t hi, int64_t lo, double scale) {
    const double a = (double)hi * 0x1p28, b = (double)lo;  // both exact
    const double sum = a + b;
    const double bb = sum - a;
    const double e = (a - (sum - bb)) + (b - bb);
    const double sv = sum * scale, ev = e * scale;
    const float r = __double2float_rn(sv);
    if (ev == 0.0 || (double)r == sv) return r;
    const float dn = __double2float_rd(sv), up = __double2float_ru(sv);
    const double mid = 0.5 * ((double)dn + (double)up);
    if (sv != mid) return r;
    return ev > 0.0 ? up : dn;
}

__device__ __forceinline__ double logit_bound(double u, int t, int i, int T,
                                              const double* __restrict__ r1,
                                              const double* __restrict__ l2,
                                              const float* __restrict__ vmax, double gamma64) {
    return r1[t] * (double)vmax[T + i] + r1[T + i] * (double)vmax[t] +
           gamma64 * l2[t] * l2[T + i] + 0x1p-52 * fabs(u) + 1e-300;
}

__global__ void __launch_bounds__(kCertWarps * 32) route_certify_kernel(
    const int32_t* __restrict__ acc, const double* __restrict__ rsc,
    const int32_t* __restrict__ rex, const double* __restrict__ r1,
    const double* __restrict__ l2, const float* __restrict__ vmax,
    const double* __restrict__ lb, const float* __restrict__ bias,
    const float* __restrict__ logit_offset, int T, int N, int n_groups, int topk_groups,
    int topk, double gamma64, int32_t* __restrict__ cand, int32_t* __restrict__ cert,
    float* __restrict__ u_exact, int32_t* __restrict__ list, int32_t* __restrict__ list_count,
    int32_t* __restrict__ pair_list, int32_t* __restrict__ pair_count, int* dev_status,
    int32_t* __restrict__ check) {
    extern __shared__ __align__(16) float cert_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // expert i at i + i / 32: the lanes of a group scan (stride ng, often 32)
    // and of a 32-wide sweep then hit distinct banks
    const int pitch = cert_pitch(N);
    float* cen = cert_smem + warp * 3 * pitch;
    float* lo = cen + pitch;
    float* hi = lo + pitch;
    const int t = blockIdx.x * kCertWarps + warp;
    if (t >= T) return;  // no block-wide barrier below
    const int64_t plane = int64_t(T) * N;
    bool fin = rex[t] >= 0;
    for (int i = lane; i < N; i += 32) {
        const double u = level_sum(acc, plane, int64_t(t) * N + i) * rsc[t] * rsc[T + i];
        const double off = logit_offset ? (double)logit_offset[i] : 0.0;
        const double b = (double)bias[i];
        const double B = logit_bound(u, t, i, T, r1, l2, vmax, gamma64);
        const double Bp = B + 0x1p-23 * (fabs(u) + fabs(off) + B);
        const double c = 1.0 / (1.0 + exp(-(u + off))) + b;
        const double delta = 0.25 * Bp + 0x1p-23 + 0x1p-24 * fabs(b) + 1e-14;
        fin = fin && rex[T + i] >= 0 && isfinite(c) && isfinite(delta);
        cen[cert_at(i)] = __double2float_rn(c);
        lo[cert_at(i)] = __double2float_rd(c - delta);
        hi[cert_at(i)] = __double2float_ru(c + delta);
    }
    fin = __all_sync(0xffffffffu, fin);
    __syncwarp();
    bool ok = fin;
    const int ng = N / n_groups;
    // group scores on the centres, and the group intervals
    float gv = -INFINITY, glo = -INFINITY, ghi = -INFINITY;
    int gi = INT_MAX;
    if (lane < n_groups) {
        for (int j = 0; j < ng; ++j) {
            const int i = lane * ng + j;
            gv = fmaxf(gv, cen[cert_at(i)]);
            glo = fmaxf(glo, lo[cert_at(i)]);
            ghi = fmaxf(ghi, hi[cert_at(i)]);
        }
        gi = lane;
    }
    uint32_t gmask = 0;
    {
        float v = gv;
        int id = gi;
        for (int r = 0; r < topk_groups; ++r) {
            float bv = v;
            int bi = id;
            warp_argmax(bv, bi);
            if (bi == INT_MAX) break;
            gmask |= 1u << bi;
            if (lane == bi) id = INT_MAX;  // taken
        }
    }
    if (topk_groups < n_groups) {
        const bool sel = lane < n_groups && ((gmask >> lane) & 1u);
        const float min_sel = warp_min(sel ? glo : INFINITY);
        const float max_rej = warp_max((lane < n_groups && !sel) ? ghi : -INFINITY);
        ok = ok && (min_sel > max_rej);
    }
    // top-K inside the chosen groups on the centres; lane owns experts
    // lane + 32j
    uint32_t taken = 0;
    int my_idx = INT_MAX;
    for (int r = 0; r < topk; ++r) {
        float bv = 0.0f;
        int bi = INT_MAX;
        for (int j = 0, i = lane; i < N; ++j, i += 32) {
            if ((taken >> j) & 1u) continue;
            if (!((gmask >> (i / ng)) & 1u)) continue;
            if (better(cen[cert_at(i)], i, bv, bi)) {
                bv = cen[cert_at(i)];
                bi = i;
            }
        }
        warp_argmax(bv, bi);
        if (bi == INT_MAX) break;
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        if (lane == r) my_idx = bi;
    }
    {
        const float chosen_lo = warp_min((lane < topk && my_idx < N) ? lo[cert_at(my_idx)] : INFINITY);
        float rej_hi = -INFINITY;
        for (int j = 0, i = lane; i < N; ++j, i += 32) {
            if ((taken >> j) & 1u) continue;
            if (!((gmask >> (i / ng)) & 1u)) continue;
            rej_hi = fmaxf(rej_hi, hi[cert_at(i)]);
        }
        rej_hi = warp_max(rej_hi);
        const bool all_chosen = __all_sync(0xffffffffu, lane >= topk || my_idx < N);
        ok = ok && all_chosen && (chosen_lo > rej_hi);
    }
    if (lane < topk) {
        cand[int64_t(t) * topk + lane] = ok ? my_idx : -1;
        if (ok) {
            int64_t hi, lo;
            level_parts(acc, plane, int64_t(t) * N + my_idx, hi, lo);
            const double scale = rsc[t] * rsc[T + my_idx];
            const double u = ((double)hi * 0x1p28 + (double)lo) * scale;
            const double B = logit_bound(u, t, my_idx, T, r1, l2, vmax, gamma64);
            const float a = __double2float_rn(u - B), z = __double2float_rn(u + B);
            if (rex[t] == 1 && rex[T + my_idx] == 1 && sum_is_exact(t, my_idx, T, l2, lb)) {
                // the levels hold the exact sum and the defining sum equals it
                u_exact[int64_t(t) * topk + lane] = exact_level_fp32(hi, lo, scale);
            } else if (a == z) {
                u_exact[int64_t(t) * topk + lane] = a;
            } else {  // to be summed: job (t, slot) on the pair list
                const int pos = atomicAdd(pair_count, 1);
                if (pos < T * topk) pair_list[pos] = t * topk + lane;
                else route_bad(dev_status, check, 0, pos);
            }
        }
    }
    if (lane == 0) {
        cert[t] = ok ? 1 : 0;
        if (!ok) {
            const int pos = atomicAdd(list_count, 1);
            if (pos < T) list[pos] = t;
            else route_bad(dev_status, check, 0, pos);
        }
    }
}

// ------------------------------------------------ 4. exact (defining) sums
// u_def = fp32 of the FP64 sum of x[t,k]*E[i,k] in ascending k.  A bf16
// value v has no bit below |v| * 2^-8, so a product of two has none below
// |x E| * 2^-16; when every nonzero |x E| of the row pair lies in
// [2^-133, 2^127) (checked from the rows' ranges) every product is exact in
// fp32, is formed there and added in FP64, which equals the FP64 fma of the
// definition.  Otherwise both factors are widened to FP64 first.
// Products of one 16-byte vector pair (8 k), widened to FP64.
__device__ __forceinline__ void vec_products(const uint4& xv, const uint4& ev, bool fp32_products,
                                             double (&p)[8]) {
    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
    const uint32_t ew[4] = {ev.x, ev.y, ev.z, ev.w};
    if (fp32_products) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            p[2 * q] = (double)__fmul_rn(bf16_lo(xw[q]), bf16_lo(ew[q]));
            p[2 * q + 1] = (double)__fmul_rn(bf16_hi(xw[q]), bf16_hi(ew[q]));
        }
    } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            p[2 * q] = __dmul_rn(bf16_lo_d(xw[q]), bf16_lo_d(ew[q]));
            p[2 * q + 1] = __dmul_rn(bf16_hi_d(xw[q]), bf16_hi_d(ew[q]));
        }
    }
}

// Chosen logits that the bound did not settle come from one sum per warp;
// every logit of the tokens on the uncertified list from one chain per
// thread while the list holds at most kPairList tokens, from the tiled
// kernel below for longer lists.
constexpr int kPairList = 256;

// Exactness of one row pair's defining sum, decided by a warp.  Every
// product p_k = x_k E_k is exact in FP64 and a multiple of 2^lowbit(p_k);
// with g the smallest lowbit over the nonzero products and S = sum |p_k|,
// every partial sum (in any order) is a multiple of 2^g of magnitude at
// most S, hence a double when S < 2^(53+g).  Then no addition of the
// defining ascending-k sum rounds and it equals the exact sum, which the
// warp forms in parallel (each lane sums its k in order, then a shuffle
// tree; every step exact).  S is accumulated rounding upward, so the test
// is rigorous.  Returns false (no result) when the test fails or a value
// is not finite.
__device__ __forceinline__ bool warp_exact_logit(const uint16_t* __restrict__ xr,
                                                 const uint16_t* __restrict__ er, int d,
                                                 int lane, float& u) {
    const uint4* xp = reinterpret_cast<const uint4*>(xr);
    const uint4* ep = reinterpret_cast<const uint4*>(er);
    constexpr int kAhead = 7;  // 16-byte vectors of each row in flight per lane
    const int nv = d / 8;
    double sabs = 0.0, sum = 0.0;
    int g = INT_MAX;
    bool finite = true;
    for (int v0 = lane; v0 < nv; v0 += 32 * kAhead) {
        // this lane's next kAhead vectors of both rows, loaded before use; past
        // the row end they are zero (zero products change no sum)
        uint4 xa[kAhead], ea[kAhead];
#pragma unroll
        for (int i = 0; i < kAhead; ++i) {
            const int v = v0 + 32 * i;
            xa[i] = v < nv ? __ldg(xp + v) : make_uint4(0u, 0u, 0u, 0u);
            ea[i] = v < nv ? __ldg(ep + v) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int i = 0; i < kAhead; ++i) {
            const uint32_t xw[4] = {xa[i].x, xa[i].y, xa[i].z, xa[i].w};
            const uint32_t ew[4] = {ea[i].x, ea[i].y, ea[i].z, ea[i].w};
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint32_t xb = q & 1 ? xw[q >> 1] >> 16 : xw[q >> 1] & 0xFFFFu;
                const uint32_t eb = q & 1 ? ew[q >> 1] >> 16 : ew[q >> 1] & 0xFFFFu;
                finite = finite && ((xb >> 7) & 0xFFu) != 0xFFu && ((eb >> 7) & 0xFFu) != 0xFFu;
                const double pk = (double)__uint_as_float(xb << 16) * (double)__uint_as_float(eb << 16);
                sabs = __dadd_ru(sabs, fabs(pk));
                sum = __dadd_rn(sum, pk);
                if (pk != 0.0) {
                    // lowest set bit of the (normal, exact) double product
                    const uint64_t bits = uint64_t(__double_as_longlong(pk));
                    const int ex = int((bits >> 52) & 0x7FFu);
                    const uint64_t sig = (bits & 0xFFFFFFFFFFFFFull) | (uint64_t(1) << 52);
                    g = min(g, ex - 1075 + (__ffsll((long long)sig) - 1));
                }
            }
        }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        sabs = __dadd_ru(sabs, __shfl_xor_sync(0xffffffffu, sabs, o));
        sum = __dadd_rn(sum, __shfl_xor_sync(0xffffffffu, sum, o));
        g = min(g, __shfl_xor_sync(0xffffffffu, g, o));
    }
    finite = __all_sync(0xffffffffu, finite);
    if (!finite) return false;
    if (g == INT_MAX) {  // every product is zero: the defining sum is +0
        u = 0.0f;
        return true;
    }
    if (!(sabs < ldexp(1.0, 53 + g))) return false;
    u = __double2float_rn(sum);
    return true;
}

// Jobs of the exact-sum kernels: the listed chosen logits (pair list).  Job
// j -> token t, expert e and the pair index pj; false when an index is out
// of range.
struct ExactJobs {
    int64_t nA;
};

__device__ __forceinline__ ExactJobs exact_jobs(int T, int K, const int32_t* pair_count,
                                                const int32_t* list_count, int* dev_status,
                                                int32_t* check, bool report) {
    int np = *pair_count, nl = *list_count;
    if (np > T * K || nl > T) {
        if (report) route_bad(dev_status, check, 1, max(np, nl));
        np = min(np, T * K);
    }
    return {int64_t(np)};
}

__device__ __forceinline__ bool exact_job(int64_t j, int T, int N, int K,
                                          const int32_t* __restrict__ cand,
                                          const int32_t* __restrict__ pair_list, int& t, int& e,
                                          int& pj) {
    pj = pair_list[j];
    t = pj / K;
    e = (pj >= 0 && pj < T * K) ? cand[pj] : -1;
    return t >= 0 && t < T && e >= 0 && e < N;
}

// Phase 1, one warp per pair-list job (a chosen logit of a certified token
// whose fp32 rounding was not settled): the warp settles the job by
// warp_exact_logit when its defining sum cannot round (nearly every row pair
// of real data) and otherwise marks it with a NaN for phase 2.  The full
// rows of uncertified tokens skip this test (route_list_rows_kernel): those
// tokens are uncertified mostly because of values far below their row's
// maximum, which also fail it.
__global__ void __launch_bounds__(64) route_exact_pairs_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ E, int T, int N, int d, int K,
    const int32_t* __restrict__ cand, const int32_t* __restrict__ pair_list,
    const int32_t* __restrict__ pair_count, const int32_t* __restrict__ list_count,
    float* __restrict__ u_exact, int* dev_status, int32_t* __restrict__ check) {
    const int lane = threadIdx.x & 31;
    const ExactJobs jobs = exact_jobs(T, K, pair_count, list_count, dev_status, check,
                                      blockIdx.x == 0 && threadIdx.x == 0);
    const int64_t stride = int64_t(gridDim.x) * (blockDim.x / 32);
    for (int64_t j = int64_t(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5); j < jobs.nA;
         j += stride) {
        int t, e, pj;
        if (!exact_job(j, T, N, K, cand, pair_list, t, e, pj)) {
            if (lane == 0) route_bad(dev_status, check, 2, int(j));
            continue;
        }
        // the reductions leave identical values in every lane: `fast` and u
        // are warp-uniform
        float u = 0.0f;
        const bool fast = warp_exact_logit(x + int64_t(t) * d, E + int64_t(e) * d, d, lane, u);
        if (lane == 0) u_exact[pj] = fast ? u : __int_as_float(0x7FFFFFFF);
    }
}

// The defining sum of one row pair by a warp, in ascending k: the lanes load
// the rows 32 vectors (256 k) per chunk, form the exact products and store
// them in a 4-chunk ring in shared memory, while lane 0 adds the chunk three
// behind in order.  The additions are the definition's own, one dependent
// chain; the warp only keeps the operands streaming (a lone thread waited
// on its loads).  Returns the fp32 result in every lane.
constexpr int kChainRing = 4;
__device__ __forceinline__ float warp_chain_logit(const uint16_t* __restrict__ xr,
                                                  const uint16_t* __restrict__ er, int d,
                                                  bool fp32_products, int lane,
                                                  double* __restrict__ ring) {
    const uint4* xp = reinterpret_cast<const uint4*>(xr);
    const uint4* ep = reinterpret_cast<const uint4*>(er);
    const int nv = d / 8;
    const int nch = (nv + 31) / 32;
    auto store = [&](int ch, const uint4& xv, const uint4& ev) {
        double p[8];
        vec_products(xv, ev, fp32_products, p);
        double* dst = ring + (ch % kChainRing) * 256 + lane * 8;
#pragma unroll
        for (int q = 0; q < 8; ++q) dst[q] = p[q];
    };
    for (int ch = 0; ch < kChainRing - 1 && ch < nch; ++ch) {
        const int v = ch * 32 + lane;
        if (v < nv) store(ch, __ldg(xp + v), __ldg(ep + v));
    }
    __syncwarp();
    double acc = 0.0;
    for (int ch = 0; ch < nch; ++ch) {
        // the loads of the chunk kChainRing - 1 ahead go out before lane 0's adds
        const int ahead = ch + kChainRing - 1;
        const int v = ahead * 32 + lane;
        uint4 xv = make_uint4(0u, 0u, 0u, 0u), ev = xv;
        if (ahead < nch && v < nv) {
            xv = __ldg(xp + v);
            ev = __ldg(ep + v);
        }
        if (lane == 0) {
            const double* src = ring + (ch % kChainRing) * 256;
            const int n = min(32, nv - ch * 32) * 8;
            for (int i = 0; i < n; ++i) acc = __dadd_rn(acc, src[i]);
        }
        // the slot of chunk `ahead` held chunk ch - 1, summed last round
        if (ahead < nch && v < nv) store(ahead, xv, ev);
        __syncwarp();
    }
    return __shfl_sync(0xffffffffu, __double2float_rn(acc), 0);
}

// Phase 2, one warp per job: the pair-list jobs phase 1 marked (NaN) get the
// defining sum in ascending k.  Settled results are never NaN: phase 1
// settles only finite row pairs.  (The listed tokens' rows go to
// route_list_rows_kernel.)
constexpr int kChainWarps = 2;
__global__ void __launch_bounds__(32 * kChainWarps) route_exact_chain_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ E, int T, int N, int d, int K,
    const int32_t* __restrict__ cand, const int32_t* __restrict__ pair_list,
    const int32_t* __restrict__ pair_count, const int32_t* __restrict__ list_count,
    const float* __restrict__ vmax, const float* __restrict__ vmin, float* __restrict__ u_exact,
    int* dev_status, int32_t* __restrict__ check) {
    __shared__ __align__(16) double ring[kChainWarps][kChainRing * 256];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const ExactJobs jobs = exact_jobs(T, K, pair_count, list_count, dev_status, check, false);
    const int64_t stride = int64_t(gridDim.x) * kChainWarps;
    for (int64_t j = int64_t(blockIdx.x) * kChainWarps + warp; j < jobs.nA; j += stride) {
        int t, e, pj;
        // (a bad pair index was reported by phase 1)
        if (!exact_job(j, T, N, K, cand, pair_list, t, e, pj)) continue;
        if (!isnan(u_exact[pj])) continue;  // settled in phase 1 (warp-uniform)
        const bool fp32_products = double(vmin[t]) * double(vmin[T + e]) >= 0x1p-133 &&
                                   double(vmax[t]) * double(vmax[T + e]) < 0x1p127;
        const float u = warp_chain_logit(x + int64_t(t) * d, E + int64_t(e) * d, d,
                                         fp32_products, lane, ring[warp]);
        if (lane == 0) u_exact[pj] = u;
    }
}

// Every logit of the listed (uncertified) tokens while the list is short:
// one thread per (listed token, expert) runs the defining sum in ascending
// k.  The bf16 x bf16 products are exact in FP64, so each FMA is the
// definition's addition of one product; where the rows' ranges keep every
// product a normal-range fp32 (the test of the chain kernel), the product is
// formed in fp32, exactly, and one conversion per term replaces two.  A block
// takes one listed token and kRowThreads experts.  A chain is d dependent
// FP64 additions, so the operands must arrive well ahead:
// asynchronous copies keep kRowStages - 1 chunks of 64 k in flight, each
// thread copying its own expert row into its slot of a shared ring and 8
// threads the token's row, which the whole block reads.
constexpr int kRowThreads = 64;
constexpr int kRowStages = 3;
constexpr int kRowChunk = 8;                    // 16-byte vectors per row and chunk
constexpr int kRowPitch = kRowChunk * 16 + 16;  // a thread's slot (padded: no bank conflicts)

__device__ __forceinline__ void row_cp16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(tc::smem_u32(dst)), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void row_cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void row_cp_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__global__ void __launch_bounds__(kRowThreads) route_list_rows_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ E, int T, int d, int n_routed,
    const int32_t* __restrict__ list, const int32_t* __restrict__ list_count,
    const float* __restrict__ vmax, const float* __restrict__ vmin, double* __restrict__ uhat,
    int* dev_status, int32_t* __restrict__ check) {
    __shared__ __align__(16) uint8_t es[kRowStages][kRowThreads * kRowPitch];
    __shared__ __align__(16) uint4 xs[kRowStages][kRowChunk];
    const int nl = min(*list_count, T);
    const int l = blockIdx.x;
    if (nl > kPairList || l >= nl) return;  // uniform over the block
    const int t = list[l];
    if (t < 0 || t >= T) {
        if (threadIdx.x == 0) route_bad(dev_status, check, 2, t);
        return;
    }
    const int tid = threadIdx.x;
    const int e = blockIdx.y * kRowThreads + tid;
    const bool e_ok = e < n_routed;  // threads past N copy nothing but keep the barriers
    const uint4* xp = reinterpret_cast<const uint4*>(x + int64_t(t) * d);
    const uint4* ep = reinterpret_cast<const uint4*>(E + int64_t(e_ok ? e : 0) * d);
    const int nv = d / 8;
    const int nch = (nv + kRowChunk - 1) / kRowChunk;
    const bool fp32_products = e_ok && double(vmin[t]) * double(vmin[T + e]) >= 0x1p-133 &&
                               double(vmax[t]) * double(vmax[T + e]) < 0x1p127;
    auto issue = [&](int ch) {
        if (ch < nch) {
            const int st = ch % kRowStages, v0 = ch * kRowChunk;
            if (e_ok) {
#pragma unroll
                for (int i = 0; i < kRowChunk; ++i)
                    if (v0 + i < nv) row_cp16(&es[st][tid * kRowPitch + 16 * i], ep + v0 + i);
            }
            if (tid < kRowChunk && v0 + tid < nv) row_cp16(&xs[st][tid], xp + v0 + tid);
        }
        row_cp_commit();  // (an empty group past the row end keeps the count)
    };
#pragma unroll
    for (int ch = 0; ch < kRowStages - 1; ++ch) issue(ch);
    double acc = 0.0;
    for (int ch = 0; ch < nch; ++ch) {
        row_cp_wait<kRowStages - 2>();  // this thread's copies of chunk ch have landed
        __syncthreads();                // so have everyone's; chunk ch - 1 is consumed
        issue(ch + kRowStages - 1);     // into the slot chunk ch - 1 held
        const int st = ch % kRowStages;
        const int nvc = min(kRowChunk, nv - ch * kRowChunk);
#pragma unroll
        for (int i = 0; i < kRowChunk; ++i) {
            if (i < nvc) {
                const uint4 xv = xs[st][i];
                const uint4 ev = *reinterpret_cast<const uint4*>(&es[st][tid * kRowPitch + 16 * i]);
                const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
                const uint32_t ew[4] = {ev.x, ev.y, ev.z, ev.w};
                if (fp32_products) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        acc = __dadd_rn(acc, (double)__fmul_rn(bf16_lo(xw[q]), bf16_lo(ew[q])));
                        acc = __dadd_rn(acc, (double)__fmul_rn(bf16_hi(xw[q]), bf16_hi(ew[q])));
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        acc = fma(bf16_lo_d(xw[q]), bf16_lo_d(ew[q]), acc);
                        acc = fma(bf16_hi_d(xw[q]), bf16_hi_d(ew[q]), acc);
                    }
                }
            }
        }
    }
    row_cp_wait<0>();
    if (e_ok) uhat[int64_t(t) * n_routed + e] = (double)__double2float_rn(acc);
}

// The same sums for a long list, in 64 x 64 tiles of (listed token, expert):
// thread (ty, tx) owns tokens 8ty..8ty+7 and experts 8tx..8tx+7 of the tile
// (64 FP64 accumulators, ascending k).  The K chunk is staged in shared
// memory as doubles, the experts interleaved (expert 8tx+j at column 8j+tx)
// so that the 8 threads of a row read consecutive doubles; chunks are
// double-buffered and the next one is fetched into registers while the
// current one is multiplied.  Does nothing while the list is short.
constexpr int kLT = 64;   // tokens per logits tile
constexpr int kLE = 64;   // experts per logits tile
constexpr int kLK = 16;   // k per smem stage (double-buffered)
constexpr int kLV = kLK / 8;  // 16-byte vectors per row and stage
constexpr int kLThreads = 64;

__global__ void __launch_bounds__(kLThreads) route_logits_list_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ E, int T, int d, int n_routed,
    const int32_t* __restrict__ list, const int32_t* __restrict__ list_count,
    double* __restrict__ uhat, int* dev_status, int32_t* __restrict__ check) {
    __shared__ __align__(16) double xs[2][kLK][kLT];
    __shared__ __align__(16) double es[2][kLK][kLE];
    const int nl = min(*list_count, T);
    const int l0 = blockIdx.x * kLT, e0 = blockIdx.y * kLE;
    if (nl <= kPairList || l0 >= nl) return;
    const int tid = threadIdx.x, ty = tid >> 3, tx = tid & 7;
    // loader: thread tid stages row tid of the x tile (listed token l0 + tid)
    // and row tid of the E tile, kLK k values of each per chunk
    const bool xrow_ok = l0 + tid < nl, erow_ok = e0 + tid < n_routed;
    int xt = xrow_ok ? list[l0 + tid] : 0;
    if (xt < 0 || xt >= T) {
        route_bad(dev_status, check, 3, xt);
        xt = 0;
    }
    const uint4* xp = reinterpret_cast<const uint4*>(x + int64_t(xt) * d);
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
                xs[buf][kk][tid] = bf16_lo_d(xw[j]);
                xs[buf][kk + 1][tid] = bf16_hi_d(xw[j]);
                es[buf][kk][ecol] = bf16_lo_d(ew[j]);
                es[buf][kk + 1][ecol] = bf16_hi_d(ew[j]);
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
        const int l = l0 + ty * 8 + i;
        if (l >= nl) continue;
        const int t = list[l];
        if (t < 0 || t >= T) continue;  // reported above
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = e0 + tx * 8 + j;
            if (e < n_routed) uhat[int64_t(t) * n_routed + e] = (double)__double2float_rn(acc[i][j]);
        }
    }
}

// ------------------------------------------------------------- 5. select
// One warp per token.  Certified token: lanes k < K hold the chosen experts
// and their exact logits; s and s' follow the definition, the slots are
// ordered by descending s' (ties to the lower expert).  Listed token: the
// full selection on its exact logits.  Gates: S = FP64 sum of the chosen s
// in slot order, gate_k = fp32(s_k / S).  Shared memory: the block
// histogram [N_r] followed by per-warp s and s' arrays [2][N_r].
constexpr int kSelWarps = 8;

__global__ void __launch_bounds__(kSelWarps * 32) route_select_kernel(
    const double* __restrict__ uhat, const int32_t* __restrict__ cert,
    const int32_t* __restrict__ cand, const float* __restrict__ u_exact, int T, int n_routed,
    int n_groups, int topk_groups, int topk, const float* __restrict__ bias,
    const float* __restrict__ logit_offset, int32_t* __restrict__ topk_idx,
    float* __restrict__ topk_gate, float* __restrict__ topk_score,
    int32_t* __restrict__ counts, int* dev_status,
    int32_t* __restrict__ check) {
    extern __shared__ __align__(16) float sel_smem[];
    int* hist = reinterpret_cast<int*>(sel_smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float* s = sel_smem + n_routed + warp * 2 * n_routed;
    float* sb = s + n_routed;
    for (int i = threadIdx.x; i < n_routed; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const int t = blockIdx.x * kSelWarps + warp;
    if (t < T) {
        int my_idx = INT_MAX;  // expert of slot `lane`
        float sv = 0.0f;       // its unbiased s
        if (cert[t]) {
            int idx = INT_MAX;
            float sbv = 0.0f, s_own = 0.0f;
            if (lane < topk) {
                idx = cand[int64_t(t) * topk + lane];
                if (idx < 0 || idx >= n_routed) {
                    route_bad(dev_status, check, 4, idx);
                    idx = 0;
                }
                float ui = u_exact[int64_t(t) * topk + lane];
                if (logit_offset) ui = __fadd_rn(ui, logit_offset[idx]);
                s_own = __double2float_rn(1.0 / (1.0 + exp(-(double)ui)));
                sbv = __fadd_rn(s_own, bias[idx]);
            }
            int key = idx;  // INT_MAX once placed
            for (int r = 0; r < topk; ++r) {
                float bv = sbv;
                int bi = key;
                warp_argmax(bv, bi);
                const int src = __ffs(__ballot_sync(0xffffffffu, key == bi && bi != INT_MAX)) - 1;
                const float s_r = __shfl_sync(0xffffffffu, s_own, src < 0 ? 0 : src);
                if (lane == src) key = INT_MAX;
                if (lane == r) {
                    my_idx = bi;
                    sv = s_r;
                }
            }
        } else {
            const double* ut = uhat + int64_t(t) * n_routed;
            for (int i = lane; i < n_routed; i += 32) {
                float ui = (float)ut[i];  // exact fp32 logit stored as a double
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
            if (lane < topk) {
                if (my_idx < 0 || my_idx >= n_routed) {
                    route_bad(dev_status, check, 5, my_idx);
                    my_idx = 0;
                }
                sv = s[my_idx];
            }
        }
        // gates: S = FP64 sum of the chosen unbiased s in slot order
        double S = 0.0;
        for (int r = 0; r < topk; ++r) S += (double)__shfl_sync(0xffffffffu, sv, r);
        if (lane < topk && (my_idx < 0 || my_idx >= n_routed)) {
            route_bad(dev_status, check, 4, my_idx);
            my_idx = 0;
        }
        if (lane < topk) {
            topk_idx[int64_t(t) * topk + lane] = my_idx;
            topk_gate[int64_t(t) * topk + lane] = __double2float_rn((double)sv / S);
            if (topk_score) topk_score[int64_t(t) * topk + lane] = sv;
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

// Workspace of moe_route: every piece starts on a 256-byte boundary.
struct RouteWs {
    int8_t* xp;          // [4, T, d]  digit planes of x
    int8_t* ep;          // [4, N, d]  digit planes of E
    int32_t* acc;        // [7, T, N]  integer levels
    double* rsc;         // [T + N]
    int32_t* rex;        // [T + N]
    double* r1;          // [T + N]
    double* l2;          // [T + N]
    float* vmax;         // [T + N]
    float* vmin;         // [T + N]
    double* lb;          // [T + N]
    double* uhat;        // [T, N]  exact logits of listed tokens
    int32_t* cand;       // [T, K]
    float* u_exact;      // [T, K]
    int32_t* cert;       // [T]
    int32_t* list;       // [T]
    int32_t* list_count; // [1]
    int32_t* pair_list;  // [T * K]
    int32_t* pair_count; // [1]
    int32_t* check;      // [kCheckWords]
    size_t bytes;
};

RouteWs route_carve(const MoeShape* s, void* base) {
    RouteWs w{};
    const size_t T = s->T, N = s->n_routed, K = s->topk, d = s->d;
    uintptr_t p = reinterpret_cast<uintptr_t>(base);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = align_up(off + bytes, 256);
        return reinterpret_cast<void*>(p + at);
    };
    w.xp = static_cast<int8_t*>(take(4 * T * d));
    w.ep = static_cast<int8_t*>(take(4 * N * d));
    w.acc = static_cast<int32_t*>(take(size_t(kLevels) * T * N * 4));
    w.rsc = static_cast<double*>(take((T + N) * 8));
    w.rex = static_cast<int32_t*>(take((T + N) * 4));
    w.r1 = static_cast<double*>(take((T + N) * 8));
    w.l2 = static_cast<double*>(take((T + N) * 8));
    w.vmax = static_cast<float*>(take((T + N) * 4));
    w.vmin = static_cast<float*>(take((T + N) * 4));
    w.lb = static_cast<double*>(take((T + N) * 8));
    w.uhat = static_cast<double*>(take(T * N * 8));
    w.cand = static_cast<int32_t*>(take(T * K * 4));
    w.u_exact = static_cast<float*>(take(T * K * 4));
    w.cert = static_cast<int32_t*>(take(T * 4));
    w.list = static_cast<int32_t*>(take(T * 4));
    w.list_count = static_cast<int32_t*>(take(4));
    w.pair_list = static_cast<int32_t*>(take(T * K * 4));
    w.pair_count = static_cast<int32_t*>(take(4));
    w.check = static_cast<int32_t*>(take(4 * kCheckWords));
    w.bytes = off;
    return w;
}

}  // namespace moe

using namespace moe;

extern "C" MOE_API size_t moe_route_workspace_size(const MoeShape* shape) {
    if (validate_shape(shape) != MOE_OK) return 0;
    return route_carve(shape, nullptr).bytes;
}

extern "C" MOE_API int moe_route_scores(const MoeShape* shape, const uint16_t* x,
                                        const uint16_t* router_w, const float* bias,
                                        const float* logit_offset, int32_t* topk_idx,
                                        float* topk_gate, float* topk_score,
                                        int32_t* expert_counts, void* ws, size_t ws_bytes,
                                        int* dev_status, void* stream) {
    int rc = validate_shape(shape);
    if (rc != MOE_OK) return rc;
    if (!router_w || !bias || !expert_counts) return MOE_ERR_NULL;
    const int T = shape->T, d = shape->d, N = shape->n_routed, K = shape->topk;
    cudaStream_t st = as_stream(stream);
    if (cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * N, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (T == 0) return check_launch();
    if (!x || !topk_idx || !topk_gate) return MOE_ERR_NULL;
    if (!aligned16(x) || !aligned16(router_w)) return MOE_ERR_ALIGN;
    if (!ws || ws_bytes < moe_route_workspace_size(shape)) return MOE_ERR_WORKSPACE;
    // every buffer the kernels touch must be addressable by the GPU (a
    // pageable host array here would fault the kernels)
    for (const void* ptr : {(const void*)x, (const void*)router_w, (const void*)bias,
                            (const void*)logit_offset, (const void*)topk_idx,
                            (const void*)topk_gate, (const void*)topk_score,
                            (const void*)expert_counts, (const void*)ws, (const void*)dev_status})
        if (!device_accessible(ptr)) return MOE_ERR_ARG;
    const RouteWs w = route_carve(shape, ws);
    const int sms = sm_count();
    if (!device_is_sm100()) return MOE_ERR_DEVICE;

    // 1. digit planes and row statistics (also clears the list counter)
    const double nmargin = 4.0 * (d + 64) * 0x1p-53 + 0x1p-50;
    const int staged = 2 * d <= kSliceStageMax;
    const size_t slice_smem = staged ? size_t(kSliceWarps) * 2 * d : 0;
    if (slice_smem > 48 * 1024 &&
        cudaFuncSetAttribute(route_slice_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(slice_smem)) != cudaSuccess)
        return MOE_ERR_CUDA;
    route_slice_kernel<<<(T + N + kSliceWarps - 1) / kSliceWarps, kSliceWarps * 32, slice_smem,
                         st>>>(x, router_w, T, N, d, nmargin, staged, w.xp, w.ep, w.rsc, w.rex,
                               w.r1, w.l2, w.vmax, w.vmin, w.lb, w.list_count, w.pair_count,
                               w.check);
    if ((rc = check_launch()) != MOE_OK) return rc;

    // 2. integer logits; K is split when the tiles alone leave SMs idle
    const int tiles = ((T + kIM - 1) / kIM) * ((N + kIN - 1) / kIN);
    const int nchunks = d / kIK;
    int splits = sms / tiles;
    if (splits > nchunks) splits = nchunks;
    if (splits < 1) splits = 1;
    const int per_split = (nchunks + splits - 1) / splits;
    splits = (nchunks + per_split - 1) / per_split;
    if (splits > 1 &&
        cudaMemsetAsync(w.acc, 0, sizeof(int32_t) * kLevels * size_t(T) * N, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    CUtensorMap mx, me;
    if (!make_map(&mx, w.xp, 4 * uint64_t(T), uint64_t(d), kIM) ||
        !make_map(&me, w.ep, 4 * uint64_t(N), uint64_t(d), kIN))
        return MOE_ERR_CUDA;
    if (cudaFuncSetAttribute(route_imma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(kImmaSmem)) != cudaSuccess)
        return MOE_ERR_CUDA;
    dim3 gi((T + kIM - 1) / kIM, (N + kIN - 1) / kIN, splits);
    route_imma_kernel<<<gi, 128, kImmaSmem, st>>>(mx, me, T, N, nchunks, per_split, w.acc,
                                                  dev_status, wait_limit_ns());
    if ((rc = check_launch()) != MOE_OK) return rc;

    // 3. certify the choice of every token; gamma_d of FP64 bounds the
    // defining sum's rounding: |u_def - sum| <= gamma_d ||x|| ||E||
    const double gamma64 = (double(d) * 0x1p-53 / (1.0 - double(d) * 0x1p-53)) * (1.0 + 0x1p-20);
    const size_t csmem = sizeof(float) * 3 * size_t(cert_pitch(N)) * kCertWarps;
    if (csmem > 48 * 1024 &&
        cudaFuncSetAttribute(route_certify_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(csmem)) != cudaSuccess)
        return MOE_ERR_CUDA;
    route_certify_kernel<<<(T + kCertWarps - 1) / kCertWarps, kCertWarps * 32, csmem, st>>>(
        w.acc, w.rsc, w.rex, w.r1, w.l2, w.vmax, w.lb, bias, logit_offset, T, N, shape->n_groups,
        shape->topk_groups, K, gamma64, w.cand, w.cert, w.u_exact, w.list, w.list_count,
        w.pair_list, w.pair_count, dev_status, w.check);
    if ((rc = check_launch()) != MOE_OK) return rc;

    // 4. the defining FP64 sums where they are needed: a warp per chosen
    // logit where the sum provably cannot round, then a warp per remaining
    // one (the ascending-k chain); the listed tokens' rows a thread per sum
    // (short list) or in tiles (long list)
    route_exact_pairs_kernel<<<unsigned(sms * 8), 64, 0, st>>>(
        x, router_w, T, N, d, K, w.cand, w.pair_list, w.pair_count, w.list_count, w.u_exact,
        dev_status, w.check);
    if ((rc = check_launch()) != MOE_OK) return rc;
    route_exact_chain_kernel<<<unsigned(sms * 8), 32 * kChainWarps, 0, st>>>(
        x, router_w, T, N, d, K, w.cand, w.pair_list, w.pair_count, w.list_count, w.vmax,
        w.vmin, w.u_exact, dev_status, w.check);
    if ((rc = check_launch()) != MOE_OK) return rc;
    if (T > 0) {
        dim3 gr(unsigned(std::min(T, kPairList)), unsigned((N + kRowThreads - 1) / kRowThreads));
        route_list_rows_kernel<<<gr, kRowThreads, 0, st>>>(x, router_w, T, d, N, w.list,
                                                           w.list_count, w.vmax, w.vmin, w.uhat,
                                                           dev_status, w.check);
        if ((rc = check_launch()) != MOE_OK) return rc;
    }
    dim3 gl((T + kLT - 1) / kLT, (N + kLE - 1) / kLE);
    route_logits_list_kernel<<<gl, kLThreads, 0, st>>>(x, router_w, T, d, N, w.list,
                                                       w.list_count, w.uhat, dev_status, w.check);
    if ((rc = check_launch()) != MOE_OK) return rc;

    // 5. slot order, gates, histogram
    const size_t smem = sizeof(float) * size_t(N) * (1 + 2 * kSelWarps);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(route_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(smem)) != cudaSuccess)
        return MOE_ERR_CUDA;
    route_select_kernel<<<(T + kSelWarps - 1) / kSelWarps, kSelWarps * 32, smem, st>>>(
        w.uhat, w.cert, w.cand, w.u_exact, T, N, shape->n_groups, shape->topk_groups, K, bias,
        logit_offset, topk_idx, topk_gate, topk_score, expert_counts, dev_status, w.check);
    return check_launch();
}

extern "C" MOE_API int moe_route(const MoeShape* shape, const uint16_t* x,
                                 const uint16_t* router_w, const float* bias,
                                 const float* logit_offset, int32_t* topk_idx, float* topk_gate,
                                 int32_t* expert_counts, void* ws, size_t ws_bytes,
                                 int* dev_status, void* stream) {
    return moe_route_scores(shape, x, router_w, bias, logit_offset, topk_idx, topk_gate, nullptr,
                            expert_counts, ws, ws_bytes, dev_status, stream);
}
