// Token-to-expert routing ("DeepSeek-V3 Technical Report" notes page,
// section "DeepSeekMoE and auxiliary-loss-free load balancing"): sigmoid
// affinity, bias for the routing decision only, group-limited top-K (the
// "at most M nodes" rule with expert groups standing in for nodes), gates
// normalised from the unbiased affinities, and the per-batch expert load
// histogram.  Gating stays in high precision (section "FP8 mixed precision
// training"): a logit is the FP64 dot product summed in ascending k, rounded
// to fp32, so the result is reproducible bit for bit.
//
// Computing all T*N_r logits that way is FP64-bound.  The path here
// computes them cheaply with a rigorous error bound, decides the routing
// from the bounds wherever they decide it, and evaluates the defining FP64
// sum only where it is needed:
//   1. route_norms_kernel: ||x_t||_2, ||E_i||_2 and the range of |values| of
//      every row;
//   2. route_approx_kernel: u~ = fp32 sums over blocks of 32 k (packed fp32
//      FMA), the block sums added in FP64.  Each product of two bf16 values
//      is exact in fp32, so |u~ - u_def| <= c * ||x_t|| * ||E_i|| + tiny,
//      c = gamma_31 (fp32) + FP64 terms (Cauchy-Schwarz on sum |x_k E_k|);
//   3. route_certify_kernel (warp per token): intervals for every biased
//      score s' from that bound (sigmoid is 1/4-Lipschitz; fp32 roundings
//      are bounded), the group / top-K choice on the interval centres, and
//      a check that every chosen interval lies strictly above every rejected
//      one.  Then the chosen set equals the set the definition chooses.
//      Tokens that fail the check go on a list;
//   4. route_exact_pairs_kernel: the defining FP64 sum for the K chosen
//      logits of every certified token and, when the list is short, for all
//      N_r logits of every listed token (one sum per thread);
//      route_logits_list_kernel does the listed tokens in 64x64 FP64 tiles
//      when the list is long;
//   5. route_select_kernel (warp per token): exact s and s' of the chosen
//      experts, slot order, gates and histogram for certified tokens; the
//      full selection on the exact logits for listed ones.
#include <float.h>
#include <math.h>

#include "common.cuh"

namespace moe {
namespace {

// --------------------------------------------------------------- helpers
// bf16 pair (one 32-bit word) -> fp32 values
__device__ __forceinline__ uint64_t pack2f(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void unpack2f(uint64_t v, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ void fma2(uint64_t& d, uint64_t a, uint64_t b) {
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(d) : "l"(a), "l"(b));
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t d;
    const uint64_t zero = 0;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(zero));
    return d;
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

// ------------------------------------------------------------ 1. row norms
// One warp per row; rows [0, T) are tokens, [T, T+N) router rows.
//   norm[r] = sqrt(sum v^2) in FP64, raised by the factor (1 + nmargin) that
//             covers its rounding;
//   vmax[r] = max |v| (+inf if the row holds a non-finite value);
//   vmin[r] = min |v| over v != 0 (FLT_MAX for an all-zero row).
// Block 0 also clears the list counter of this call.
__global__ void __launch_bounds__(256) route_norms_kernel(const uint16_t* __restrict__ x,
                                                          const uint16_t* __restrict__ E, int T,
                                                          int N, int d, double nmargin,
                                                          double* __restrict__ norm,
                                                          float* __restrict__ vmax,
                                                          float* __restrict__ vmin,
                                                          int32_t* __restrict__ list_count) {
    if (blockIdx.x == 0 && threadIdx.x == 0) *list_count = 0;
    const int lane = threadIdx.x & 31;
    const int warps = gridDim.x * (blockDim.x >> 5);
    for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < T + N; r += warps) {
        const uint4* row = reinterpret_cast<const uint4*>(r < T ? x + int64_t(r) * d
                                                                : E + int64_t(r - T) * d);
        double ss = 0.0;
        float mx = 0.0f, mn = FLT_MAX;
        for (int v = lane; v < d / 8; v += 32) {
            const uint4 w = __ldg(row + v);
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float f = h ? bf16_hi(ws[q]) : bf16_lo(ws[q]);
                    const float a = fabsf(f);
                    mx = (a <= FLT_MAX) ? fmaxf(mx, a) : INFINITY;
                    if (a > 0.0f) mn = fminf(mn, a);
                    ss = fma((double)f, (double)f, ss);
                }
            }
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            ss += __shfl_xor_sync(0xffffffffu, ss, o);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        }
        if (lane == 0) {
            norm[r] = sqrt(ss) * (1.0 + nmargin);
            vmax[r] = mx;
            vmin[r] = mn;
        }
    }
}

// -------------------------------------------------------- 2. approx logits
// Tile of 32 tokens x 32 experts per CTA of one warp; lane (ty, tx) =
// (lane / 4, lane % 4) owns tokens 4ty..4ty+3 and experts 8tx..8tx+7.  K is
// walked in blocks of 32: the block's x and E slices are staged in shared
// memory as fp32 (x duplicated into pairs for the packed FMA), the block
// sum starts from the exact first product and takes 31 packed fp32 FMAs,
// and is then added to an FP64 accumulator.  blockIdx.z splits K into
// gridDim.z ranges of whole blocks; with more than one range the partial
// sums are added atomically (any order: only the bound matters here).
constexpr int kAT = 32, kAE = 32, kAK = 32;

__global__ void __launch_bounds__(32) route_approx_kernel(const uint16_t* __restrict__ x,
                                                          const uint16_t* __restrict__ E, int T,
                                                          int N, int d, int blocks_per_split,
                                                          double* __restrict__ uhat) {
    __shared__ __align__(16) uint64_t xs[kAK][kAT];  // (x, x) pairs
    __shared__ __align__(16) float es[kAK][kAE];
    const int lane = threadIdx.x, ty = lane >> 2, tx = lane & 3;
    const int t0 = blockIdx.x * kAT, e0 = blockIdx.y * kAE;
    const int nblk = d / kAK;
    const int b0 = blockIdx.z * blocks_per_split;
    const int b1 = min(nblk, b0 + blocks_per_split);
    if (b0 >= b1) return;
    // loader: lane stages x row t0 + lane and router row e0 + lane
    const bool xrow_ok = t0 + lane < T, erow_ok = e0 + lane < N;
    const uint4* xp = reinterpret_cast<const uint4*>(x + int64_t(t0 + lane) * d);
    const uint4* ep = reinterpret_cast<const uint4*>(E + int64_t(e0 + lane) * d);
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    uint4 xv[4], ev[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        xv[i] = xrow_ok ? __ldg(xp + b0 * 4 + i) : zero;
        ev[i] = erow_ok ? __ldg(ep + b0 * 4 + i) : zero;
    }
    double acc64[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc64[i][j] = 0.0;
    for (int b = b0; b < b1; ++b) {
        __syncwarp();  // the previous block's reads of the tile are done
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t xw[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
            const uint32_t ew[4] = {ev[i].x, ev[i].y, ev[i].z, ev[i].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int kk = 8 * i + 2 * j;
                const float xl = bf16_lo(xw[j]), xh = bf16_hi(xw[j]);
                xs[kk][lane] = pack2f(xl, xl);
                xs[kk + 1][lane] = pack2f(xh, xh);
                es[kk][lane] = bf16_lo(ew[j]);
                es[kk + 1][lane] = bf16_hi(ew[j]);
            }
        }
        __syncwarp();
        if (b + 1 < b1) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                xv[i] = xrow_ok ? __ldg(xp + (b + 1) * 4 + i) : zero;
                ev[i] = erow_ok ? __ldg(ep + (b + 1) * 4 + i) : zero;
            }
        }
        uint64_t acc[4][4];
#pragma unroll
        for (int k = 0; k < kAK; ++k) {
            const ulonglong2 xa = *reinterpret_cast<const ulonglong2*>(&xs[k][4 * ty]);
            const ulonglong2 xb = *reinterpret_cast<const ulonglong2*>(&xs[k][4 * ty + 2]);
            const ulonglong2 ea = *reinterpret_cast<const ulonglong2*>(&es[k][8 * tx]);
            const ulonglong2 eb = *reinterpret_cast<const ulonglong2*>(&es[k][8 * tx + 4]);
            const uint64_t xr[4] = {xa.x, xa.y, xb.x, xb.y};
            const uint64_t er[4] = {ea.x, ea.y, eb.x, eb.y};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (k == 0) acc[i][j] = mul2(xr[i], er[j]);
                    else fma2(acc[i][j], xr[i], er[j]);
                }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float a, c;
                unpack2f(acc[i][j], a, c);
                acc64[i][2 * j] += (double)a;
                acc64[i][2 * j + 1] += (double)c;
            }
    }
    const bool split = gridDim.z > 1;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = t0 + 4 * ty + i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = e0 + 8 * tx + j;
            if (e >= N) continue;
            double* dst = uhat + int64_t(t) * N + e;
            if (split) atomicAdd(dst, acc64[i][j]);
            else *dst = acc64[i][j];
        }
    }
}

// ---------------------------------------------------------- 3. certify
// One warp per token.  For expert i, with u~ the approximation and
//   B  = cbound * ||x_t|| * ||E_i|| + 2^-23 |u~| + tiny   (>= |u~ - u_def|),
// the biased score s'_i of the definition lies within delta_i of
// centre_i = sigma(u~ + off_i) + b_i, where
//   delta_i = B'/4 + 2^-23 + 2^-24 |b_i| + 1e-14,
//   B' = B + 2^-23 (|u~| + |off_i| + B)
// (B' covers the two fp32 roundings of u and of u + off; sigma is
// 1/4-Lipschitz; 2^-23 + 2^-24 |b_i| covers the fp32 roundings of s and
// s + b; 1e-14 the FP64 evaluation of sigma).  The interval ends are stored
// rounded outwards to fp32.  Groups and experts are chosen on the centres;
// the choice is certified when the lowest chosen lower end is strictly above
// the highest rejected upper end, for the groups and then for the experts
// inside the chosen groups.
constexpr int kCertWarps = 8;

__global__ void __launch_bounds__(kCertWarps * 32) route_certify_kernel(
    const double* __restrict__ uhat, const double* __restrict__ norm,
    const float* __restrict__ bias, const float* __restrict__ logit_offset, int T, int N,
    int n_groups, int topk_groups, int topk, double cbound, double tiny,
    int32_t* __restrict__ cand, int32_t* __restrict__ cert, int32_t* __restrict__ list,
    int32_t* __restrict__ list_count) {
    extern __shared__ __align__(16) float cert_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float* cen = cert_smem + warp * 3 * N;
    float* lo = cen + N;
    float* hi = lo + N;
    const int t = blockIdx.x * kCertWarps + warp;
    if (t >= T) return;  // no block-wide barrier below
    const double nx = norm[t];
    bool fin = true;
    for (int i = lane; i < N; i += 32) {
        const double u = uhat[int64_t(t) * N + i];
        const double off = logit_offset ? (double)logit_offset[i] : 0.0;
        const double b = (double)bias[i];
        const double B = cbound * nx * norm[T + i] + 0x1p-23 * fabs(u) + tiny;
        const double Bp = B + 0x1p-23 * (fabs(u) + fabs(off) + B);
        const double c = 1.0 / (1.0 + exp(-(u + off))) + b;
        const double delta = 0.25 * Bp + 0x1p-23 + 0x1p-24 * fabs(b) + 1e-14;
        fin = fin && isfinite(c) && isfinite(delta);
        cen[i] = __double2float_rn(c);
        lo[i] = __double2float_rd(c - delta);
        hi[i] = __double2float_ru(c + delta);
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
            gv = fmaxf(gv, cen[i]);
            glo = fmaxf(glo, lo[i]);
            ghi = fmaxf(ghi, hi[i]);
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
            if (better(cen[i], i, bv, bi)) {
                bv = cen[i];
                bi = i;
            }
        }
        warp_argmax(bv, bi);
        if (bi == INT_MAX) break;
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        if (lane == r) my_idx = bi;
    }
    {
        const float chosen_lo = warp_min((lane < topk && my_idx < N) ? lo[my_idx] : INFINITY);
        float rej_hi = -INFINITY;
        for (int j = 0, i = lane; i < N; ++j, i += 32) {
            if ((taken >> j) & 1u) continue;
            if (!((gmask >> (i / ng)) & 1u)) continue;
            rej_hi = fmaxf(rej_hi, hi[i]);
        }
        rej_hi = warp_max(rej_hi);
        const bool all_chosen = __all_sync(0xffffffffu, lane >= topk || my_idx < N);
        ok = ok && all_chosen && (chosen_lo > rej_hi);
    }
    if (lane < topk) cand[int64_t(t) * topk + lane] = ok ? my_idx : -1;
    if (lane == 0) {
        cert[t] = ok ? 1 : 0;
        if (!ok) list[atomicAdd(list_count, 1)] = t;
    }
}

// ------------------------------------------------ 4. exact (defining) sums
// u_def = fp32 of the FP64 sum of x[t,k]*E[i,k] in ascending k.  A bf16
// value v has no bit below |v| * 2^-8, so a product of two has none below
// |x E| * 2^-16; when every nonzero |x E| of the row pair lies in
// [2^-133, 2^127) (checked from the rows' ranges) every product is exact in
// fp32, is formed there and added in FP64, which equals the FP64 fma of the
// definition.  Otherwise both factors are widened to FP64 first.
__device__ __forceinline__ float exact_logit(const uint16_t* __restrict__ xr,
                                             const uint16_t* __restrict__ er, int d,
                                             bool fp32_products) {
    const uint4* xp = reinterpret_cast<const uint4*>(xr);
    const uint4* ep = reinterpret_cast<const uint4*>(er);
    const int nv = d / 8;
    double acc = 0.0;
    uint4 xa = __ldg(xp), ea = __ldg(ep);
    for (int v = 0; v < nv; ++v) {
        uint4 xb = xa, eb = ea;
        if (v + 1 < nv) {
            xb = __ldg(xp + v + 1);
            eb = __ldg(ep + v + 1);
        }
        const uint32_t xw[4] = {xa.x, xa.y, xa.z, xa.w};
        const uint32_t ew[4] = {ea.x, ea.y, ea.z, ea.w};
        if (fp32_products) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                acc = __dadd_rn(acc, (double)__fmul_rn(bf16_lo(xw[q]), bf16_lo(ew[q])));
                acc = __dadd_rn(acc, (double)__fmul_rn(bf16_hi(xw[q]), bf16_hi(ew[q])));
            }
        } else {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                acc = __fma_rn(bf16_lo_d(xw[q]), bf16_lo_d(ew[q]), acc);
                acc = __fma_rn(bf16_hi_d(xw[q]), bf16_hi_d(ew[q]), acc);
            }
        }
        xa = xb;
        ea = eb;
    }
    return __double2float_rn(acc);
}

// Tokens on the uncertified list get every logit from one sum per thread
// while the list holds at most kPairList tokens; longer lists go to the
// tiled kernel below.
constexpr int kPairList = 256;

__global__ void __launch_bounds__(256) route_exact_pairs_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ E, int T, int N, int d, int K,
    const int32_t* __restrict__ cand, const int32_t* __restrict__ cert,
    const int32_t* __restrict__ list, const int32_t* __restrict__ list_count,
    const float* __restrict__ vmax, const float* __restrict__ vmin,
    float* __restrict__ u_exact, double* __restrict__ uhat) {
    const int64_t nA = int64_t(T) * K;
    const int nl = *list_count;
    const int64_t nB = nl <= kPairList ? int64_t(nl) * N : 0;
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t j = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; j < nA + nB; j += stride) {
        int t, e;
        if (j < nA) {
            t = int(j / K);
            if (!cert[t]) continue;
            e = cand[j];
        } else {
            const int64_t jj = j - nA;
            t = list[jj / N];
            e = int(jj % N);
        }
        const bool fp32_products = double(vmin[t]) * double(vmin[T + e]) >= 0x1p-133 &&
                                   double(vmax[t]) * double(vmax[T + e]) < 0x1p127;
        const float u = exact_logit(x + int64_t(t) * d, E + int64_t(e) * d, d, fp32_products);
        if (j < nA) u_exact[j] = u;
        else uhat[int64_t(t) * N + e] = (double)u;
    }
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
    double* __restrict__ uhat) {
    __shared__ __align__(16) double xs[2][kLK][kLT];
    __shared__ __align__(16) double es[2][kLK][kLE];
    const int nl = *list_count;
    const int l0 = blockIdx.x * kLT, e0 = blockIdx.y * kLE;
    if (nl <= kPairList || l0 >= nl) return;
    const int tid = threadIdx.x, ty = tid >> 3, tx = tid & 7;
    // loader: thread tid stages row tid of the x tile (listed token l0 + tid)
    // and row tid of the E tile, kLK k values of each per chunk
    const bool xrow_ok = l0 + tid < nl, erow_ok = e0 + tid < n_routed;
    const int xt = xrow_ok ? list[l0 + tid] : 0;
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
    float* __restrict__ topk_gate, int32_t* __restrict__ counts) {
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
            if (lane < topk) sv = s[my_idx];
        }
        // gates: S = FP64 sum of the chosen unbiased s in slot order
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

// Workspace of moe_route: every piece starts on a 256-byte boundary.
struct RouteWs {
    double* uhat;        // [T, N]  approximate, then exact for listed tokens
    double* norm;        // [T + N]
    float* vmax;         // [T + N]
    float* vmin;         // [T + N]
    int32_t* cand;       // [T, K]
    float* u_exact;      // [T, K]
    int32_t* cert;       // [T]
    int32_t* list;       // [T]
    int32_t* list_count; // [1]
    size_t bytes;
};

RouteWs route_carve(const MoeShape* s, void* base) {
    RouteWs w{};
    const size_t T = s->T, N = s->n_routed, K = s->topk;
    uintptr_t p = reinterpret_cast<uintptr_t>(base);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = align_up(off + bytes, 256);
        return reinterpret_cast<void*>(p + at);
    };
    w.uhat = static_cast<double*>(take(T * N * 8));
    w.norm = static_cast<double*>(take((T + N) * 8));
    w.vmax = static_cast<float*>(take((T + N) * 4));
    w.vmin = static_cast<float*>(take((T + N) * 4));
    w.cand = static_cast<int32_t*>(take(T * K * 4));
    w.u_exact = static_cast<float*>(take(T * K * 4));
    w.cert = static_cast<int32_t*>(take(T * 4));
    w.list = static_cast<int32_t*>(take(T * 4));
    w.list_count = static_cast<int32_t*>(take(4));
    w.bytes = off;
    return w;
}

}  // namespace moe

using namespace moe;

extern "C" MOE_API size_t moe_route_workspace_size(const MoeShape* shape) {
    if (validate_shape(shape) != MOE_OK) return 0;
    return route_carve(shape, nullptr).bytes;
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
    const int T = shape->T, d = shape->d, N = shape->n_routed, K = shape->topk;
    cudaStream_t st = as_stream(stream);
    if (cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * N, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (T == 0) return check_launch();
    if (!x || !topk_idx || !topk_gate) return MOE_ERR_NULL;
    if (!aligned16(x) || !aligned16(router_w)) return MOE_ERR_ALIGN;
    if (!ws || ws_bytes < moe_route_workspace_size(shape)) return MOE_ERR_WORKSPACE;
    const RouteWs w = route_carve(shape, ws);
    const int sms = sm_count();

    // 1. norms and ranges of every row (also clears the list counter)
    const double nmargin = 4.0 * (d + 64) * 0x1p-53 + 0x1p-50;
    route_norms_kernel<<<(T + N + 7) / 8, 256, 0, st>>>(x, router_w, T, N, d, nmargin, w.norm,
                                                        w.vmax, w.vmin, w.list_count);
    if ((rc = check_launch()) != MOE_OK) return rc;

    // 2. approximate logits; K is split when the tiles alone fill few SMs
    const int tiles = ((T + kAT - 1) / kAT) * ((N + kAE - 1) / kAE);
    const int nblk = d / kAK;
    int splits = (4 * sms + tiles - 1) / tiles;
    if (splits > nblk) splits = nblk;
    if (splits < 1) splits = 1;
    const int per_split = (nblk + splits - 1) / splits;
    splits = (nblk + per_split - 1) / per_split;
    if (splits > 1 &&
        cudaMemsetAsync(w.uhat, 0, sizeof(double) * size_t(T) * N, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    dim3 ga((T + kAT - 1) / kAT, (N + kAE - 1) / kAE, splits);
    route_approx_kernel<<<ga, 32, 0, st>>>(x, router_w, T, N, d, per_split, w.uhat);
    if ((rc = check_launch()) != MOE_OK) return rc;

    // 3. certify the choice of every token
    // |u~ - u_def| <= cbound * ||x|| ||E|| + tiny: gamma_31 of fp32 for the
    // block sums, FP64 terms for the sum of block sums and for the defining
    // FP64 sum, products below 2^-126 (at most 2^-150 off each) in tiny.
    const double u32 = 0x1p-24;
    const double cbound = (31.0 * u32 / (1.0 - 31.0 * u32)) * (1.0 + 0x1p-20) +
                          4.0 * (d + nblk + 64) * 0x1p-53;
    const double tiny = double(d) * 0x1p-148;
    const size_t csmem = sizeof(float) * 3 * size_t(N) * kCertWarps;
    if (csmem > 48 * 1024 &&
        cudaFuncSetAttribute(route_certify_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(csmem)) != cudaSuccess)
        return MOE_ERR_CUDA;
    route_certify_kernel<<<(T + kCertWarps - 1) / kCertWarps, kCertWarps * 32, csmem, st>>>(
        w.uhat, w.norm, bias, logit_offset, T, N, shape->n_groups, shape->topk_groups, K,
        cbound, tiny, w.cand, w.cert, w.list, w.list_count);
    if ((rc = check_launch()) != MOE_OK) return rc;

    // 4. the defining FP64 sums where they are needed
    int64_t pair_threads = int64_t(T) * K + int64_t(kPairList) * N;
    int64_t pblocks = (pair_threads + 255) / 256;
    if (pblocks > int64_t(sms) * 16) pblocks = int64_t(sms) * 16;
    route_exact_pairs_kernel<<<unsigned(pblocks), 256, 0, st>>>(
        x, router_w, T, N, d, K, w.cand, w.cert, w.list, w.list_count, w.vmax, w.vmin,
        w.u_exact, w.uhat);
    if ((rc = check_launch()) != MOE_OK) return rc;
    dim3 gl((T + kLT - 1) / kLT, (N + kLE - 1) / kLE);
    route_logits_list_kernel<<<gl, kLThreads, 0, st>>>(x, router_w, T, d, N, w.list,
                                                       w.list_count, w.uhat);
    if ((rc = check_launch()) != MOE_OK) return rc;

    // 5. slot order, gates, histogram
    const size_t smem = sizeof(float) * size_t(N) * (1 + 2 * kSelWarps);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(route_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(smem)) != cudaSuccess)
        return MOE_ERR_CUDA;
    route_select_kernel<<<(T + kSelWarps - 1) / kSelWarps, kSelWarps * 32, smem, st>>>(
        w.uhat, w.cert, w.cand, w.u_exact, T, N, shape->n_groups, shape->topk_groups, K, bias,
        logit_offset, topk_idx, topk_gate, expert_counts);
    return check_launch();
}
