/*
 * CPU oracle for the DeepSeekMoE layer forward with FP8 block scaling.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check and the CPU
 * baseline of the benchmark may load this library.  It shares no code,
 * header, table or constant generator with the CUDA library, and the CUDA
 * library never calls it.
 *
 * Plain, slow, obviously correct: every step follows the definition in
 * "DeepSeek-V3 Technical Report" (notes page), sections "DeepSeekMoE and
 * auxiliary-loss-free load balancing" and "FP8 mixed precision training".
 * Floating point is FP64 unless the method fixes a storage precision (FP32
 * scores, gates, scales and bias; E4M3 codes; bf16 inputs).
 *
 * Readings of the pages that this file fixes (the pages leave them open):
 *   Q  scale = fp32(amax / 448); inv = fp32(448 / amax); code =
 *      E4M3(fp32(v * inv)) rounded to nearest even and clamped to +-448;
 *      amax = 0 gives scale 1 and codes +-0.
 *   R1 router logit u = fp32(sum over k of x*E), the sum taken in FP64 in
 *      ascending k (each bf16*bf16 product is exact in FP64).
 *   R2 s = fp32(1 / (1 + exp(-u))) in FP64; biased s' = fp32(s + b).
 *   R3 group j holds experts [j*n_g, (j+1)*n_g); group score = max s' in the
 *      group; the M best groups win, ties to the lower group index.
 *   R4 top-K by s' among experts of the chosen groups, ties to the lower
 *      expert index; output slots in the order picked.
 *   R5 gate_k = fp32(s_k / S), S = FP64 sum of the K unbiased s in slot order.
 *   R6 expert i is overloaded when count_i * N_r > T*K, underloaded when
 *      count_i * N_r < T*K; b -= gamma / b += gamma in fp32; equal: unchanged.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fPIC -shared -lm.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ bf16 */
static float bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* ------------------------------------------------------------------ E4M3 */
/* OCP FP8 E4M3 ("FN"): 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits;
 * exponent field 0 is subnormal (m * 2^-9); S.1111.111 is NaN; no infinity;
 * largest finite value 1.75 * 2^8 = 448.  The pages name the format only
 * ("E4M3 for all tensors"); its bit layout is the public OCP standard. */
double orc_e4m3_decode(uint8_t c) {
    int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* Round-to-nearest-even onto the E4M3 grid, then clamp to the largest finite
 * magnitude (saturating).  Works in FP64, where every step is exact: |v| is
 * scaled by a power of two so the grid step becomes 1 and rint() (default
 * rounding mode: nearest, ties to even) picks the neighbour. */
uint8_t orc_e4m3_encode(float v) {
    if (isnan(v)) return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    double step;
    if (a >= ldexp(1.0, -6)) {
        int e = ilogb(a);               /* floor(log2 a), a finite or inf */
        if (isinf(a)) return sign | 0x7E;
        step = ldexp(1.0, e - 3);       /* 3 mantissa bits */
    } else {
        step = ldexp(1.0, -9);          /* subnormal spacing */
    }
    double r = rint(a / step) * step;
    if (r > 448.0) r = 448.0;
    if (r == 0.0) return sign;
    int ex, mant;
    if (r < ldexp(1.0, -6)) {
        ex = 0;
        mant = (int)(r / ldexp(1.0, -9));
    } else {
        ex = ilogb(r);
        mant = (int)((r / ldexp(1.0, ex) - 1.0) * 8.0);
        ex += 7;
    }
    return (uint8_t)(sign | (ex << 3) | mant);
}

void orc_e4m3_encode_array(const float* v, int64_t n, uint8_t* out) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(v[i]);
}

/* One quantisation group: amax over its values, fp32 scale and inverse,
 * codes of fp32(v * inv).  vals holds the group's values widened to fp32. */
static float quant_group(const float* vals, int n, uint8_t* codes_out) {
    float amax = 0.0f;
    for (int i = 0; i < n; ++i) {
        float a = fabsf(vals[i]);
        if (a > amax) amax = a;
    }
    if (amax == 0.0f) {
        for (int i = 0; i < n; ++i) codes_out[i] = signbit(vals[i]) ? 0x80 : 0x00;
        return 1.0f;
    }
    float scale = amax / 448.0f;   /* fp32 division, correctly rounded */
    float inv = 448.0f / amax;
    for (int i = 0; i < n; ++i) {
        float p = vals[i] * inv;   /* fp32 product */
        codes_out[i] = orc_e4m3_encode(p);
    }
    return scale;
}

/* 1x128 tiles along the columns ("tile-wise, activations 1x128").
 * x: bf16 [rows, cols]; q: [rows, cols]; scales: [rows, cols/128]. */
void orc_quant_act_1x128_bf16(const uint16_t* x, int64_t rows, int64_t cols,
                              uint8_t* q, float* scales) {
    int64_t nt = cols / 128;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        float vals[128];
        for (int64_t t = 0; t < nt; ++t) {
            const uint16_t* src = x + r * cols + t * 128;
            for (int i = 0; i < 128; ++i) vals[i] = bf16_to_f32(src[i]);
            scales[r * nt + t] = quant_group(vals, 128, q + r * cols + t * 128);
        }
    }
}

/* Same rule on fp32 input (the SwiGLU output h, rounded to fp32). */
void orc_quant_act_1x128_f32(const float* x, int64_t rows, int64_t cols,
                             uint8_t* q, float* scales) {
    int64_t nt = cols / 128;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t t = 0; t < nt; ++t)
            scales[r * nt + t] = quant_group(x + r * cols + t * 128, 128,
                                             q + r * cols + t * 128);
}

/* 128x128 blocks ("block-wise, weights 128x128").
 * w: bf16 [rows, cols]; q: [rows, cols]; scales: [rows/128, cols/128]. */
void orc_quant_w_128x128(const uint16_t* w, int64_t rows, int64_t cols,
                         uint8_t* q, float* scales) {
    int64_t br = rows / 128, bc = cols / 128;
    #pragma omp parallel for schedule(static) collapse(2)
    for (int64_t i = 0; i < br; ++i)
        for (int64_t j = 0; j < bc; ++j) {
            float* vals = (float*)malloc(128 * 128 * sizeof(float));
            uint8_t* codes = (uint8_t*)malloc(128 * 128);
            for (int r = 0; r < 128; ++r)
                for (int c = 0; c < 128; ++c)
                    vals[r * 128 + c] = bf16_to_f32(w[(i * 128 + r) * cols + j * 128 + c]);
            scales[i * bc + j] = quant_group(vals, 128 * 128, codes);
            for (int r = 0; r < 128; ++r)
                memcpy(q + (i * 128 + r) * cols + j * 128, codes + r * 128, 128);
            free(vals);
            free(codes);
        }
}

/* ---------------------------------------- power-of-two scales (option)
 * A numerically different option, not the pages' recipe: the scale of a
 * tile or block is a power of two, so that block-scaled tensor-core MMAs
 * (UE8M0 scale factors, one byte: the exponent + 127) can apply it in the
 * MMA itself.  With amax = max |v| of the group:
 *   e = the smallest integer with amax <= 448 * 2^e (so no code saturates),
 *   clamped to [-127, 127]; amax = 0 gives e = 0;
 *   code = E4M3(v * 2^-e), nearest even, saturating (the product is exact).
 * Returns e. */
static int pow2_exponent(float amax) {
    if (!(amax > 0.0f)) return 0;
    const double a = amax;
    int e = ilogb(a) - 9;               /* 448 * 2^e < 2^(e+9) <= a: too small */
    while (a > ldexp(448.0, e)) ++e;    /* at most two steps */
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

static int quant_group_pow2(const float* vals, int n, uint8_t* codes_out) {
    float amax = 0.0f;
    for (int i = 0; i < n; ++i) {
        float a = fabsf(vals[i]);
        if (a > amax) amax = a;
    }
    const int e = pow2_exponent(amax);
    for (int i = 0; i < n; ++i)
        codes_out[i] = orc_e4m3_encode((float)ldexp((double)vals[i], -e));
    return e;
}

/* 1x128 tiles with power-of-two scales; e_out [rows, cols/128] (int32). */
void orc_quant_act_1x128_pow2_bf16(const uint16_t* x, int64_t rows, int64_t cols,
                                   uint8_t* q, int32_t* e_out) {
    int64_t nt = cols / 128;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        float vals[128];
        for (int64_t t = 0; t < nt; ++t) {
            const uint16_t* src = x + r * cols + t * 128;
            for (int i = 0; i < 128; ++i) vals[i] = bf16_to_f32(src[i]);
            e_out[r * nt + t] = quant_group_pow2(vals, 128, q + r * cols + t * 128);
        }
    }
}

void orc_quant_act_1x128_pow2_f32(const float* x, int64_t rows, int64_t cols,
                                  uint8_t* q, int32_t* e_out) {
    int64_t nt = cols / 128;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t t = 0; t < nt; ++t)
            e_out[r * nt + t] = quant_group_pow2(x + r * cols + t * 128, 128,
                                                 q + r * cols + t * 128);
}

/* 128x128 blocks with power-of-two scales; e_out [rows/128, cols/128]. */
void orc_quant_w_128x128_pow2(const uint16_t* w, int64_t rows, int64_t cols,
                              uint8_t* q, int32_t* e_out) {
    int64_t br = rows / 128, bc = cols / 128;
    #pragma omp parallel for schedule(static) collapse(2)
    for (int64_t i = 0; i < br; ++i)
        for (int64_t j = 0; j < bc; ++j) {
            float* vals = (float*)malloc(128 * 128 * sizeof(float));
            uint8_t* codes = (uint8_t*)malloc(128 * 128);
            for (int r = 0; r < 128; ++r)
                for (int c = 0; c < 128; ++c)
                    vals[r * 128 + c] = bf16_to_f32(w[(i * 128 + r) * cols + j * 128 + c]);
            e_out[i * bc + j] = quant_group_pow2(vals, 128 * 128, codes);
            for (int r = 0; r < 128; ++r)
                memcpy(q + (i * 128 + r) * cols + j * 128, codes + r * 128, 128);
            free(vals);
            free(codes);
        }
}

/* ---------------------------------------------------------------- routing */
/* Sigmoid affinity, bias-adjusted group-limited top-K, normalised gates and
 * the per-expert load histogram ("DeepSeekMoE and auxiliary-loss-free load
 * balancing").  logit_offset (nullable) adds a fixed per-expert fp32 prior to
 * the logits (used only to make a skewed workload).
 * Outputs: topk_idx/topk_gate [T,K]; counts [N_r] (overwritten);
 * logits/scores (nullable) [T,N_r]: u and s for the self-checks. */
int orc_route(int T, int d, int n_routed, int n_groups, int topk_groups, int topk,
              const uint16_t* x, const uint16_t* router_w, const float* bias,
              const float* logit_offset, int32_t* topk_idx, float* topk_gate,
              int32_t* counts, float* logits_out, float* scores_out) {
    if (n_routed % n_groups) return -1;
    int ng = n_routed / n_groups;
    if (topk_groups * ng < topk || topk_groups > n_groups) return -1;
    #pragma omp parallel
    {
        float* s = (float*)malloc(n_routed * sizeof(float));
        float* sb = (float*)malloc(n_routed * sizeof(float));
        float* gscore = (float*)malloc(n_groups * sizeof(float));
        char* gsel = (char*)malloc(n_groups);
        char* esel = (char*)malloc(n_routed);
        #pragma omp for schedule(dynamic, 4)
        for (int t = 0; t < T; ++t) {
            const uint16_t* xt = x + (int64_t)t * d;
            for (int i = 0; i < n_routed; ++i) {
                const uint16_t* ei = router_w + (int64_t)i * d;
                double acc = 0.0;
                for (int k = 0; k < d; ++k)
                    acc += (double)bf16_to_f32(xt[k]) * (double)bf16_to_f32(ei[k]);
                float u = (float)acc;
                if (logit_offset) u = u + logit_offset[i];
                float si = (float)(1.0 / (1.0 + exp(-(double)u)));
                s[i] = si;
                sb[i] = si + bias[i];
                if (logits_out) logits_out[(int64_t)t * n_routed + i] = u;
                if (scores_out) scores_out[(int64_t)t * n_routed + i] = si;
            }
            /* group scores and the M best groups */
            for (int g = 0; g < n_groups; ++g) {
                float m = sb[g * ng];
                for (int j = 1; j < ng; ++j)
                    if (sb[g * ng + j] > m) m = sb[g * ng + j];
                gscore[g] = m;
                gsel[g] = 0;
            }
            for (int r = 0; r < topk_groups; ++r) {
                int best = -1;
                for (int g = 0; g < n_groups; ++g)
                    if (!gsel[g] && (best < 0 || gscore[g] > gscore[best])) best = g;
                gsel[best] = 1;
            }
            /* top-K experts inside the chosen groups */
            memset(esel, 0, n_routed);
            double S = 0.0;
            for (int r = 0; r < topk; ++r) {
                int best = -1;
                for (int i = 0; i < n_routed; ++i)
                    if (gsel[i / ng] && !esel[i] && (best < 0 || sb[i] > sb[best])) best = i;
                esel[best] = 1;
                topk_idx[(int64_t)t * topk + r] = best;
            }
            for (int r = 0; r < topk; ++r) S += (double)s[topk_idx[(int64_t)t * topk + r]];
            for (int r = 0; r < topk; ++r)
                topk_gate[(int64_t)t * topk + r] =
                    (float)((double)s[topk_idx[(int64_t)t * topk + r]] / S);
        }
        free(s); free(sb); free(gscore); free(gsel); free(esel);
    }
    for (int i = 0; i < n_routed; ++i) counts[i] = 0;
    for (int64_t p = 0; p < (int64_t)T * topk; ++p) counts[topk_idx[p]]++;
    return 0;
}

/* Bias update b_i -/+ gamma from the batch's load (reading R6). */
void orc_update_bias(int T, int n_routed, int topk, const int32_t* counts,
                     float gamma, float* bias) {
    int64_t total = (int64_t)T * topk;
    for (int i = 0; i < n_routed; ++i) {
        int64_t c = (int64_t)counts[i] * n_routed;
        if (c > total) bias[i] = bias[i] - gamma;
        else if (c < total) bias[i] = bias[i] + gamma;
    }
}

/* Expert-contiguous layout of the routed pairs.  offsets [N_r+2]: expert e's
 * rows are [offsets[e], offsets[e+1]); the shared expert's T rows follow at
 * offsets[N_r].  row_of_pair[t,k] = offsets[e] + (number of tokens t' < t
 * routed to e), i.e. tokens keep their order inside an expert. */
void orc_permute_layout(int T, int n_routed, int topk, const int32_t* topk_idx,
                        const int32_t* counts, int32_t* offsets, int32_t* row_of_pair) {
    offsets[0] = 0;
    for (int e = 0; e < n_routed; ++e) offsets[e + 1] = offsets[e] + counts[e];
    offsets[n_routed + 1] = offsets[n_routed] + T;
    int32_t* seen = (int32_t*)calloc(n_routed, sizeof(int32_t));
    for (int t = 0; t < T; ++t)
        for (int k = 0; k < topk; ++k) {
            int e = topk_idx[(int64_t)t * topk + k];
            row_of_pair[(int64_t)t * topk + k] = offsets[e] + seen[e];
            seen[e]++;
        }
    free(seen);
}
