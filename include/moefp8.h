/*
 * moefp8 — DeepSeekMoE layer forward with FP8 block scaling, for NVIDIA B200
 * (sm_100a).  Plain C ABI: raw pointers, sizes and a CUDA stream handle.
 *
 * The method is the MoE layer of "DeepSeek-V3 Technical Report" (notes page):
 *   - section "DeepSeekMoE and auxiliary-loss-free load balancing": sigmoid
 *     token-to-expert affinity, a per-expert bias b_i added for the routing
 *     decision only, gates from the normalised selected (unbiased)
 *     affinities, 1 shared + N_r routed experts, K routed experts per token,
 *     tokens limited to M nodes (expert groups here), batch-wise expert load
 *     monitoring with b_i -/+ gamma, no token dropping;
 *   - section "FP8 mixed precision training": every GEMM input in E4M3 with
 *     fine-grained scales (1x128 activation tiles, 128x128 weight blocks)
 *     computed online from the current max |value|; FP32 accumulation;
 *     gating kept in high precision;
 *   - section "DualPipe": the dispatch / MLP / combine stages of a MoE
 *     block, here on one GPU (dispatch = an expert-contiguous permutation,
 *     combine = the gate-weighted sum).
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE pointers to caller-owned memory unless a name
 *     ends in _host.  The library allocates no device memory; scratch space
 *     comes from the caller (ws / ws_bytes).
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL =
 *     the legacy default stream).  No call synchronises the host, except
 *     moe_read_status().
 *   - The return value is a status: MOE_OK (0) or a negative MOE_ERR_*.
 *     Argument errors are detected on the host before anything is enqueued;
 *     MOE_ERR_CUDA reports a failed launch (cudaGetLastError).
 *   - dev_status (nullable) is a device int the kernels set to a positive
 *     MOE_DEV_* code when they detect a problem at run time (a bounded wait
 *     that ran out, an index or offset out of range).  The first code
 *     written wins; the caller zeroes it.
 *   - bf16 tensors are passed as uint16_t bit patterns.  E4M3 codes are
 *     uint8_t (OCP E4M3FN: bias 7, max 448, no infinities).
 *   - Scale rule (online quantisation): per group of values, amax = max|v|,
 *     scale = fp32(amax / 448), code = E4M3(fp32(v * fp32(448 / amax))),
 *     round-to-nearest-even, saturating to +-448; amax = 0 gives scale 1.
 *     A group whose amax is below 448 / FLT_MAX (about 1.3e-36) is outside
 *     the supported range.
 *   - Thread safety: the library keeps no state between calls; concurrent
 *     calls on different buffers are independent.
 *   - Bounded waits: every wait of a kernel on an mbarrier (TMA loads, MMA
 *     completion, hand-overs between warps) gives up after a limit, 2 s by
 *     default, sets MOE_DEV_TIMEOUT and lets the kernel unwind (work already
 *     in flight is waited for, TMEM is freed); the context stays usable.
 *     The environment variable MOEFP8_WAIT_LIMIT_NS (read at every call)
 *     sets another limit in nanoseconds (at least 1000).
 *   - Fault injection for tests of that path: MOEFP8_FAULT=gemm_producer
 *     (read at every call) makes the single-CTA grouped GEMM's TMA producer
 *     withhold the loads of its first stage, so that the MMA issuer's wait
 *     on that stage runs out.  Nothing faults or hangs; the call's results
 *     are garbage and dev_status reads MOE_DEV_TIMEOUT.  Unset in normal use.
 */
#ifndef MOEFP8_H
#define MOEFP8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_API __attribute__((visibility("default")))

/* host-side status codes */
#define MOE_OK 0
#define MOE_ERR_NULL -1        /* a required pointer is NULL */
#define MOE_ERR_SHAPE -2       /* a size is not a supported multiple / range */
#define MOE_ERR_ROUTE -3       /* routing shape inconsistent (N_r % G, M*n_g < K, ...) */
#define MOE_ERR_CUDA -4        /* a CUDA launch or runtime call failed */
#define MOE_ERR_ALIGN -5       /* a pointer is not 16-byte aligned */
#define MOE_ERR_WORKSPACE -6   /* ws is NULL or smaller than required */
#define MOE_ERR_ARG -7         /* another invalid argument (epilogue, flags) */
#define MOE_ERR_DEVICE -8      /* the current device is not sm_100 */
#define MOE_ERR_STATIC_LIMIT -9 /* shape too large for moe_permute_static_ws */

/* device status codes (written to *dev_status by kernels) */
#define MOE_DEV_TIMEOUT 1      /* a bounded wait inside a kernel ran out */
#define MOE_DEV_BAD_INPUT 2    /* an index or offset array was out of range; the
                                  offending entries were skipped */

/* epilogues of moe_grouped_gemm_fp8 */
#define MOE_EPI_F32 0           /* out: float [max_rows, n] */
#define MOE_EPI_BF16 1          /* out: bf16  [max_rows, n] */
#define MOE_EPI_SWIGLU_QUANT 2  /* out: E4M3 h [max_rows, n/2] + fp32 scales */

/* Shape of one MoE layer.
 *   T           tokens in the batch (>= 0)
 *   d           hidden size (multiple of 128)
 *   n_routed    routed experts N_r (1..1024)
 *   n_groups    expert groups G (N_r % G == 0, G <= 32); group j holds
 *               experts [j*N_r/G, (j+1)*N_r/G)
 *   topk_groups M, groups a token may use (1..G)
 *   topk        K, routed experts per token (1..32, K <= M*N_r/G)
 *   inter       expert intermediate size I (multiple of 128)
 *   gamma       bias update step
 * The shared expert is expert index N_r in every per-expert array. */
typedef struct {
    int T, d, n_routed, n_groups, topk_groups, topk, inter;
    float gamma;
} MoeShape;

/* Library version (major*10000 + minor*100 + patch). */
MOE_API int moe_version(void);

/* Human-readable text of a status code (static string). */
MOE_API const char* moe_status_string(int status);

/* Copy *dev_status to *host_status after synchronising `stream`.  The only
 * call that blocks the host. */
MOE_API int moe_read_status(const int* dev_status, int* host_status, void* stream);

/* ---------------------------------------------------------------- routing
 * moe_route: router logits, sigmoid affinity, bias, group-limited top-K,
 * normalised gates and the load histogram ("DeepSeekMoE and
 * auxiliary-loss-free load balancing"; gating in high precision per "FP8
 * mixed precision training").
 *   x            bf16 [T, d] row-major
 *   router_w     bf16 [N_r, d] row-major (one centroid per routed expert)
 *   bias         fp32 [N_r], read only
 *   logit_offset fp32 [N_r] or NULL: a fixed prior added to every token's
 *                logits (used to build skewed workloads; NULL = none)
 *   topk_idx     int32 [T, K] out: chosen experts, by descending biased score
 *   topk_gate    fp32 [T, K] out: gates, sum to 1 per token
 *   expert_counts int32 [N_r] out: tokens per expert (zeroed by the call)
 *   ws, ws_bytes scratch of at least moe_route_workspace_size(shape) bytes
 * Definition (bit-exact contract):
 *   u  = fp32(sum_k x[t,k]*E[i,k]) with the sum taken in FP64 in ascending k,
 *        then u = fp32(u + logit_offset[i]) when an offset is given;
 *   s  = fp32(1/(1+exp(-u))) evaluated in FP64;  s' = fp32(s + b_i);
 *   group score = max s' in the group; the M best groups are kept (ties to
 *   the lower group); the K best s' inside them are chosen (ties to the lower
 *   expert); gate_k = fp32(s_k / S) with S the FP64 sum of the chosen s in
 *   slot order.
 * Errors: MOE_ERR_NULL, MOE_ERR_SHAPE (d % 128, T < 0, N_r range),
 * MOE_ERR_ROUTE, MOE_ERR_ALIGN (x, router_w not 16-byte aligned),
 * MOE_ERR_WORKSPACE, MOE_ERR_ARG (a pointer the GPU cannot address, e.g.
 * pageable host memory), MOE_ERR_DEVICE (not sm_100), MOE_ERR_CUDA;
 * MOE_DEV_TIMEOUT or MOE_DEV_BAD_INPUT on dev_status (may be NULL).
 * The logits are computed exactly on the tensor cores from int8 digit
 * planes of x and E wherever a rigorous bound settles the result, and with
 * the defining FP64 sum elsewhere; the outputs equal the definition. */
MOE_API size_t moe_route_workspace_size(const MoeShape* shape);
MOE_API int moe_route(const MoeShape* shape, const uint16_t* x, const uint16_t* router_w,
                      const float* bias, const float* logit_offset, int32_t* topk_idx,
                      float* topk_gate, int32_t* expert_counts, void* ws, size_t ws_bytes,
                      int* dev_status, void* stream);

/* moe_route_scores: moe_route that also writes topk_score fp32 [T, K]: the
 * unbiased affinity s of each chosen expert, in slot order (the values the
 * gates are normalised from; the backward pass needs them). */
MOE_API int moe_route_scores(const MoeShape* shape, const uint16_t* x, const uint16_t* router_w,
                             const float* bias, const float* logit_offset, int32_t* topk_idx,
                             float* topk_gate, float* topk_score, int32_t* expert_counts,
                             void* ws, size_t ws_bytes, int* dev_status, void* stream);

/* ----------------------------------------------------------- quantisation
 * fp8_quant_act_1x128: online 1x128 tile quantisation of activations
 * ("FP8 mixed precision training", fine-grained quantisation).
 *   x       bf16 [rows, cols] row-major, cols % 128 == 0, 16-byte aligned
 *   q       uint8 [rows, cols] out, E4M3 codes
 *   scales  fp32 out: scales_kb_major == 0 -> [rows, cols/128];
 *           scales_kb_major == 1 -> [cols/128, rows] (the layout the
 *           grouped GEMM reads)
 * Bit-exact contract: the scale rule in the header comment. */
MOE_API int fp8_quant_act_1x128(const uint16_t* x, int64_t rows, int64_t cols, uint8_t* q,
                                float* scales, int scales_kb_major, int* dev_status,
                                void* stream);

/* fp8_quant_w_128x128: online 128x128 block quantisation of weights
 * ("FP8 mixed precision training", block-wise 128x128 for weights).
 *   w       bf16 [rows, cols] row-major, rows % 128 == 0, cols % 128 == 0
 *   q       uint8 [rows, cols] out
 *   scales  fp32 [rows/128, cols/128] out
 * Stacked expert matrices ([E*rows_e, cols]) may be passed in one call when
 * rows_e % 128 == 0: blocks never straddle experts. */
MOE_API int fp8_quant_w_128x128(const uint16_t* w, int64_t rows, int64_t cols, uint8_t* q,
                                float* scales, int* dev_status, void* stream);

/* ------------------------------------------------------------ permutation
 * moe_permute: the single-GPU "dispatch": copies every token's FP8 row once
 * per chosen expert plus once for the shared expert into an
 * expert-contiguous buffer ("DualPipe": all-to-all dispatch of FP8
 * activations, "FP8 mixed precision training": low-precision communication).
 *   topk_idx, expert_counts   as produced by moe_route
 *   xq, xs                    codes [T, d] and row-major scales [T, d/128]
 *   xq_perm                   uint8 [T*K + T, d] out
 *   xs_perm                   fp32 [d/128, T*K + T] out (kb-major)
 *   expert_offsets            int32 [N_r + 2] out: expert e owns rows
 *                             [off[e], off[e+1]); off[N_r] = T*K and the
 *                             shared expert owns [T*K, T*K + T) in token order
 *   row_of_pair               int32 [T, K] out: row of (token t, slot k);
 *                             inside an expert, tokens keep ascending order
 *   ws, ws_bytes              scratch of moe_permute_workspace_size(shape)
 * Bit-exact contract: offsets, row_of_pair and the copied bytes/scales. */
MOE_API size_t moe_permute_workspace_size(const MoeShape* shape);
MOE_API int moe_permute(const MoeShape* shape, const int32_t* topk_idx,
                        const int32_t* expert_counts, const uint8_t* xq, const float* xs,
                        uint8_t* xq_perm, float* xs_perm, int32_t* expert_offsets,
                        int32_t* row_of_pair, void* ws, size_t ws_bytes, int* dev_status,
                        void* stream);

/* moe_quant_permute: fp8_quant_act_1x128 of x fused with moe_permute.  The
 * token rows are read once in bf16 and each 1x128 tile is quantised (same
 * scale rule and rounding as fp8_quant_act_1x128) straight into the K + 1
 * destination rows, so the unpermuted codes are never written to memory
 * ("FP8 mixed precision training": activations are quantised online, per
 * 1x128 tile, before they are dispatched).
 *   x                         bf16 [T, d] (16-byte aligned)
 *   other arguments           as moe_permute (ws of moe_permute_workspace_size)
 * Bit-exact contract: equal to fp8_quant_act_1x128 followed by moe_permute.
 * Errors: as moe_permute. */
MOE_API int moe_quant_permute(const MoeShape* shape, const uint16_t* x, const int32_t* topk_idx,
                              const int32_t* expert_counts, uint8_t* xq_perm, float* xs_perm,
                              int32_t* expert_offsets, int32_t* row_of_pair, void* ws,
                              size_t ws_bytes, int* dev_status, void* stream);

/* moe_permute_static_ws: moe_permute for callers that cannot allocate
 * device memory while they run (a serving loop whose memory budget is fixed
 * at start-up, a host framework that owns all device memory through its own
 * pool); it needs no workspace argument.  The pages have no counterpart:
 * this is a property of the library, not of the method.
 *   Arguments, layouts and results are those of moe_permute, without ws.
 *   Scratch: a 1 MiB array of device memory inside the library, held by every
 *   GPU that loads the library until the process exits.  Limit:
 *   ceil(T / 64) * N_r <= 262144 (e.g. T <= 65536 with N_r = 256); larger
 *   shapes return MOE_ERR_STATIC_LIMIT without doing anything.
 *   The first call on a device looks the array's device address up (once
 *   per device and CUDA context, with that device current), so make that
 *   first call before any stream capture.  After cudaDeviceReset the next
 *   call sees a new context and looks the address up again (so make it
 *   outside a capture too).
 *   All calls share the one array: two calls whose work overlaps on the GPU
 *   (different streams, or different host threads, on one device) race and
 *   give wrong results.  Each call overwrites every scratch entry it reads,
 *   so nothing carries over from the previous call. */
MOE_API int moe_permute_static_ws(const MoeShape* shape, const int32_t* topk_idx,
                                  const int32_t* expert_counts, const uint8_t* xq,
                                  const float* xs, uint8_t* xq_perm, float* xs_perm,
                                  int32_t* expert_offsets, int32_t* row_of_pair,
                                  int* dev_status, void* stream);

/* ------------------------------------------------------------ expert GEMM
 * moe_grouped_gemm_fp8: per group g, rows [off[g], off[g+1]) of A times the
 * group's weight matrix, FP8 E4M3 operands with block scales applied on the
 * FP32 accumulator once per 128-element K block ("FP8 mixed precision
 * training": fine-grained scales, increased accumulation precision).
 *   n_groups       number of groups (>= 1); group_offsets int32 [n_groups+1]
 *                  on the device, non-decreasing, off[n_groups] <= max_rows
 *   max_rows       rows allocated in a, a_scales and out
 *   a              uint8 [max_rows, k] E4M3 codes (16-byte aligned)
 *   a_scales       fp32 [k/128, max_rows] (kb-major 1x128 scales)
 *   k              contraction size, multiple of 128
 *   w              uint8 [n_groups, n, k] E4M3 codes, K-major (row j of
 *                  group g is output feature j)
 *   w_scales       fp32 [n_groups, n/128, k/128]
 *   n              output features, multiple of 128 (of 256 for SwiGLU)
 *   epilogue:
 *     MOE_EPI_F32          out = float [max_rows, n]
 *     MOE_EPI_BF16         out = bf16  [max_rows, n] (round to nearest even)
 *     MOE_EPI_SWIGLU_QUANT rows [0, n/2) of each weight matrix are the gate
 *                          projection W1 and rows [n/2, n) the up projection
 *                          W3; h = silu(gate) * up in fp32 is quantised 1x128
 *                          along its n/2 features: out = uint8 [max_rows, n/2],
 *                          out_scales = fp32 [n/2/128, max_rows] (kb-major)
 * Rows of A outside every group are neither read into results nor written.
 * Kernel forms (moe_grouped_gemm_form tells which one a call uses): single
 * CTAs (the default), 128 tokens x 256 output columns each (128 when
 * n % 256 != 0); or, when the environment variable MOEFP8_GEMM_PAIR=1 is
 * set and n % 256 == 0, CTA pairs on two SMs (tcgen05 cta_group::2), 256
 * tokens x 256 columns per pair, each CTA loading one of the two 128-row
 * weight blocks.  Both forms apply the same per-K-block promotion; results
 * agree to fp32 accumulation order.
 * Errors: MOE_ERR_NULL, MOE_ERR_SHAPE, MOE_ERR_ARG, MOE_ERR_ALIGN,
 * MOE_ERR_DEVICE, MOE_ERR_CUDA; MOE_DEV_TIMEOUT on dev_status. */
MOE_API int moe_grouped_gemm_fp8(int n_groups, const int32_t* group_offsets, int max_rows,
                                 const uint8_t* a, const float* a_scales, int k,
                                 const uint8_t* w, const float* w_scales, int n, int epilogue,
                                 void* out, float* out_scales, int* dev_status, void* stream);

/* ------------------------------------------- power-of-two scale option
 * A numerically different option beside the pages' recipe (whose scales
 * are arbitrary FP32 values): every 1x128 tile / 128x128 block gets the
 * scale 2^e with e the smallest integer such that amax <= 448 * 2^e
 * (clamped to [-127, 127]; amax = 0 gives e = 0), stored as one UE8M0 byte
 * e + 127, and codes E4M3(v * 2^-e) (nearest even, saturating; the product
 * is exact).  The pages wish for hardware support of tile / block scaling
 * (section "FP8 mixed precision training", discussion): B200's block-scaled
 * MMA (tcgen05.mma kind::mxf8f6f4.block_scale) applies such scales inside
 * the tensor core, so the GEMM needs no per-K-block promotion.
 *
 * fp8_quant_act_1x128_ue8m0: as fp8_quant_act_1x128 with power-of-two
 *   scales; sf uint8 [rows, cols/128] (sf_kb_major = 0) or [cols/128, rows]
 *   (sf_kb_major = 1, the layout moe_grouped_gemm_mxfp8 reads).
 * fp8_quant_w_128x128_ue8m0: as fp8_quant_w_128x128; sf uint8
 *   [rows/128, cols/128].
 * Bit-exact contract: codes and scale bytes as the rule above. */
MOE_API int fp8_quant_act_1x128_ue8m0(const uint16_t* x, int64_t rows, int64_t cols,
                                      uint8_t* q, uint8_t* sf, int sf_kb_major,
                                      int* dev_status, void* stream);
MOE_API int fp8_quant_w_128x128_ue8m0(const uint16_t* w, int64_t rows, int64_t cols,
                                      uint8_t* q, uint8_t* sf, int* dev_status, void* stream);

/* moe_grouped_gemm_mxfp8: moe_grouped_gemm_fp8 for operands quantised with
 * power-of-two scales: the scales are applied by the tensor core (one UE8M0
 * byte per 32 elements of K, each 1x128 tile's byte repeated over its four
 * 32-element pieces) and the whole K range accumulates in one FP32 TMEM
 * accumulator per 128 x 256 output tile.
 *   a_sf       uint8 [k/128, max_rows] (kb-major)
 *   w_sf       uint8 [n_groups, n/128, k/128]
 *   n          a multiple of 256
 *   epilogue   MOE_EPI_F32, MOE_EPI_BF16, or MOE_EPI_SWIGLU_QUANT (h =
 *              silu(gate) * up quantised 1x128 with power-of-two scales:
 *              out uint8 [max_rows, n/2], out_sf uint8 [n/2/128, max_rows])
 * Other arguments, layouts and errors as moe_grouped_gemm_fp8. */
MOE_API int moe_grouped_gemm_mxfp8(int n_groups, const int32_t* group_offsets, int max_rows,
                                   const uint8_t* a, const uint8_t* a_sf, int k,
                                   const uint8_t* w, const uint8_t* w_sf, int n, int epilogue,
                                   void* out, uint8_t* out_sf, int* dev_status, void* stream);

/* moe_grouped_gemm_fp8_indexed: moe_grouped_gemm_fp8 where group g uses
 * weight matrix group_weight[g] (device int32 [n_groups], each in
 * [0, n_weights)) of w [n_weights, n, k] and w_scales [n_weights, n/128,
 * k/128], so that several groups can share one expert's weights (redundant
 * experts).  An index out of range is reported (MOE_DEV_BAD_INPUT) and
 * matrix 0 is used.  Other arguments as moe_grouped_gemm_fp8. */
MOE_API int moe_grouped_gemm_fp8_indexed(int n_groups, const int32_t* group_offsets,
                                         const int32_t* group_weight, int n_weights,
                                         int max_rows, const uint8_t* a, const float* a_scales,
                                         int k, const uint8_t* w, const float* w_scales, int n,
                                         int epilogue, void* out, float* out_scales,
                                         int* dev_status, void* stream);

/* moe_quant_permute_ue8m0: moe_quant_permute with power-of-two scales:
 * xsf_perm uint8 [d/128, T*K + T] (kb-major UE8M0 bytes) replaces xs_perm.
 * Bit-exact contract: equal to fp8_quant_act_1x128_ue8m0 followed by the
 * permutation of moe_permute. */
MOE_API int moe_quant_permute_ue8m0(const MoeShape* shape, const uint16_t* x,
                                    const int32_t* topk_idx, const int32_t* expert_counts,
                                    uint8_t* xq_perm, uint8_t* xsf_perm,
                                    int32_t* expert_offsets, int32_t* row_of_pair, void* ws,
                                    size_t ws_bytes, int* dev_status, void* stream);

/* --------------------------------------------------- expert parallelism
 * Dispatch and combine across P ranks ("DualPipe": all-to-all dispatch and
 * combine around the expert MLP, tokens sent to at most M nodes; "FP8 mixed
 * precision training": FP8 dispatch).  Rank q owns routed experts
 * [q E, (q+1) E), E = N_r / P (N_r % P == 0, P <= 32); every rank runs the
 * shared expert on its own tokens.  A token travels once to each rank owning
 * one of its K experts, as one row of moe_ep_row_bytes(shape) bytes:
 *   codes uint8 [d] | 1x128 scales fp32 [d/128] | local expert of each slot
 *   int32 [K] (-1: the slot's expert is on another rank) | gate of each slot
 *   fp32 [K] | source token int32 | zero padding to a multiple of 16 bytes.
 * The exchanges (row counts, rows, fp32 partial outputs) are the caller's
 * all-to-alls (NCCL); these calls build and consume the buffers.  All
 * buffers are device memory; shape->T is this rank's token count.
 *
 * moe_ep_workspace_size: scratch for moe_ep_dispatch_plan (max_recv_rows
 *   = 0) or moe_ep_local_permute (max_recv_rows = its n_recv).
 * moe_ep_dispatch_plan: from topk_idx [T, K] (moe_route): send_counts int32
 *   [P] (rows for each rank), send_offsets int32 [P + 1], send_row int32
 *   [T, P] (row of (token, rank) in the send buffer, destination-major with
 *   tokens ascending; -1 when not sent).
 * moe_ep_pack: x bf16 [T, d] quantised 1x128 (the scale rule of
 *   fp8_quant_act_1x128) into send_buf [sum send_counts, row_bytes].
 * moe_ep_local_permute: n_recv received rows -> expert-contiguous FP8 rows of
 *   the local experts: xq_perm uint8 [max_rows, d], xs_perm fp32 [d/128,
 *   max_rows] (kb-major), local_offsets int32 [E + 1], pair_row int32
 *   [n_recv, K] (local row of each slot, -1 for other ranks' slots).  Local
 *   rows keep the received order inside an expert.  Slots past max_rows are
 *   dropped and reported (MOE_DEV_BAD_INPUT); n_recv * min(K, E) rows always
 *   suffice.
 * moe_ep_partial_combine: back_buf fp32 [n_recv, d]: per received row, the
 *   sum over its local slots of gate * expert_out[pair_row] (slot order,
 *   fp32).  expert_out is moe_grouped_gemm_fp8's fp32 output over the local
 *   rows.
 * moe_ep_final_combine: y bf16 [T, d] = shared_out [T, d] (the shared
 *   expert's fp32 output) + the partial outputs back_recv [sum send_counts,
 *   d] of the token's destinations in rank order (back_recv laid out like
 *   the send buffer), rounded once to bf16.
 * Errors: MOE_ERR_ARG (P out of range or not dividing N_r), MOE_ERR_NULL,
 * MOE_ERR_SHAPE, MOE_ERR_ALIGN, MOE_ERR_WORKSPACE, MOE_ERR_CUDA. */
MOE_API size_t moe_ep_row_bytes(const MoeShape* shape);
MOE_API size_t moe_ep_workspace_size(const MoeShape* shape, int n_ranks, int max_recv_rows);
MOE_API int moe_ep_dispatch_plan(const MoeShape* shape, int n_ranks, const int32_t* topk_idx,
                                 int32_t* send_counts, int32_t* send_offsets,
                                 int32_t* send_row, void* ws, size_t ws_bytes, int* dev_status,
                                 void* stream);
MOE_API int moe_ep_pack(const MoeShape* shape, int n_ranks, const uint16_t* x,
                        const int32_t* topk_idx, const float* topk_gate,
                        const int32_t* send_row, uint8_t* send_buf, int* dev_status,
                        void* stream);
MOE_API int moe_ep_local_permute(const MoeShape* shape, int n_ranks, const uint8_t* recv_buf,
                                 int n_recv, uint8_t* xq_perm, float* xs_perm, int max_rows,
                                 int32_t* local_offsets, int32_t* pair_row, void* ws,
                                 size_t ws_bytes, int* dev_status, void* stream);
MOE_API int moe_ep_partial_combine(const MoeShape* shape, int n_ranks, const uint8_t* recv_buf,
                                   int n_recv, const int32_t* pair_row, const float* expert_out,
                                   float* back_buf, int* dev_status, void* stream);
MOE_API int moe_ep_final_combine(const MoeShape* shape, int n_ranks, const float* shared_out,
                                 const float* back_recv, const int32_t* send_row, uint16_t* y,
                                 int* dev_status, void* stream);

/* ------------------------------------------------------ redundant experts
 * The most loaded experts get extra copies so that their rows can be split
 * over several groups (618zxw.cn news article on DeepSeek-V3, redundant
 * experts for inference load balance).  On one GPU the copies share the
 * expert's weights (moe_grouped_gemm_fp8_indexed); every output row is
 * computed exactly as without copies.
 *
 * moe_plan_redundant_experts (HOST memory, synchronous): distributes
 * n_extra extra slots over n_experts experts with loads counts[e] (e.g. the
 * expert_counts of a batch): each extra slot goes to the expert with the
 * largest rows per copy ceil(counts[e] / replicas[e]) (ties to the lower
 * expert), which minimises the largest rows per copy.
 *   replicas    int32 [n_experts] out: copies per expert (>= 1)
 *   slot_expert int32 [n_experts + n_extra] out: the expert of each slot,
 *               experts ascending, an expert's copies adjacent
 * Errors: MOE_ERR_NULL, MOE_ERR_SHAPE (n_experts + n_extra + 1 > 1040),
 * MOE_ERR_ARG (a negative count).
 *
 * moe_split_groups (device): the group table of the copies.  Expert e's rows
 * [off[e], off[e+1]) of the permutation are cut into replicas[e] consecutive
 * pieces whose sizes differ by at most one (the first ones longer).
 *   expert_offsets  int32 [N_r + 2] from moe_permute / moe_quant_permute
 *   replicas, slot_expert   as planned above (device copies)
 *   first_slot      int32 [N_r] first slot of each expert (device)
 *   slot_offsets    int32 [N_r + n_extra + 2] out: group s owns rows
 *                   [slot_offsets[s], slot_offsets[s+1]); the last group is
 *                   the shared expert's rows
 *   slot_weight     int32 [N_r + n_extra + 1] out: weight matrix of each
 *                   group (slot_expert, then N_r for the shared expert) */
MOE_API int moe_plan_redundant_experts(const int32_t* counts, int n_experts, int n_extra,
                                       int32_t* replicas, int32_t* slot_expert);
MOE_API int moe_split_groups(const MoeShape* shape, const int32_t* expert_offsets,
                             const int32_t* replicas, const int32_t* slot_expert,
                             const int32_t* first_slot, int n_extra, int32_t* slot_offsets,
                             int32_t* slot_weight, int* dev_status, void* stream);

/* moe_grouped_gemm_form: CTAs per tile (1 = single CTAs, 2 = CTA pairs) that
 * moe_grouped_gemm_fp8 uses on the current device for these arguments (same
 * meaning as there), or 0 when they are invalid.  Host-only query; launches
 * nothing. */
MOE_API int moe_grouped_gemm_form(int n_groups, int max_rows, int n, int epilogue);

/* ---------------------------------------------------------------- combine
 * moe_combine: y[t] = o[shared row of t] + sum_k gate[t,k] * o[row_of_pair
 * [t,k]], accumulated in fp32 in slot order, rounded once to bf16
 * ("DualPipe": all-to-all combine, here a local gather).
 *   expert_out  fp32 [T*K + T, d] (moe_grouped_gemm_fp8 with MOE_EPI_F32)
 *   y           bf16 [T, d] out */
MOE_API int moe_combine(const MoeShape* shape, const float* expert_out,
                        const int32_t* expert_offsets, const int32_t* row_of_pair,
                        const float* topk_gate, uint16_t* y, int* dev_status, void* stream);

/* ------------------------------------------------------------ bias update
 * moe_update_bias: b_i = fp32(b_i - gamma) when count_i * N_r > T*K
 * (overloaded), fp32(b_i + gamma) when count_i * N_r < T*K (underloaded),
 * unchanged when equal ("DeepSeekMoE and auxiliary-loss-free load
 * balancing").  bias fp32 [N_r] is updated in place. */
MOE_API int moe_update_bias(const MoeShape* shape, const int32_t* expert_counts, float* bias,
                            int* dev_status, void* stream);

/* ------------------------------------------------------------ whole layer
 * Expert weights, pre-quantised with fp8_quant_w_128x128:
 *   w13        uint8 [N_r+1, 2I, d]: rows [0,I) = W1 (gate), [I,2I) = W3 (up)
 *   w13_scales fp32  [N_r+1, 2I/128, d/128]
 *   w2         uint8 [N_r+1, d, I]  (down projection, K-major)
 *   w2_scales  fp32  [N_r+1, d/128, I/128]
 *   router_w   bf16  [N_r, d]
 * Expert N_r is the shared expert. */
typedef struct {
    const uint8_t* w13;
    const float* w13_scales;
    const uint8_t* w2;
    const float* w2_scales;
    const uint16_t* router_w;
} MoeWeights;

/* Routing results of one layer call (caller-owned device buffers). */
typedef struct {
    int32_t* topk_idx;        /* [T, K] */
    float* topk_gate;         /* [T, K] */
    int32_t* expert_counts;   /* [N_r] */
    int32_t* expert_offsets;  /* [N_r + 2] */
    int32_t* row_of_pair;     /* [T, K] */
} MoeRouting;

/* moe_layer_forward: route -> quantise x (1x128) + permute (one pass,
 * moe_quant_permute) -> grouped GEMM
 * (W13, SwiGLU + 1x128 quantisation of h) -> grouped GEMM (W2, fp32) ->
 * combine -> (optionally) bias update, all on `stream`.
 *   x            bf16 [T, d];  y bf16 [T, d] out
 *   bias         fp32 [N_r]; updated in place after routing when
 *                update_bias != 0 (the next call routes with the new bias)
 *   logit_offset fp32 [N_r] or NULL (see moe_route)
 *   ws, ws_bytes scratch of moe_layer_workspace_size(shape) bytes */
MOE_API size_t moe_layer_workspace_size(const MoeShape* shape);
MOE_API int moe_layer_forward(const MoeShape* shape, const MoeWeights* weights,
                              const uint16_t* x, float* bias, const float* logit_offset,
                              MoeRouting* routing, uint16_t* y, int update_bias, void* ws,
                              size_t ws_bytes, int* dev_status, void* stream);

/* moe_layer_forward_host: the same layer with x and y in HOST memory (pinned
 * memory makes the copies asynchronous).  x_host is copied into the
 * workspace, y is copied back to y_host, both on `stream`; the caller
 * synchronises `stream` before reading y_host.
 *   ws, ws_bytes scratch of moe_layer_host_workspace_size(shape) bytes */
MOE_API size_t moe_layer_host_workspace_size(const MoeShape* shape);
MOE_API int moe_layer_forward_host(const MoeShape* shape, const MoeWeights* weights,
                                   const uint16_t* x_host, float* bias,
                                   const float* logit_offset, MoeRouting* routing,
                                   uint16_t* y_host, int update_bias, void* ws,
                                   size_t ws_bytes, int* dev_status, void* stream);

/* The whole layer with the power-of-two scale option: weights quantised
 * with fp8_quant_w_128x128_ue8m0, x and h with power-of-two 1x128 scales,
 * both expert GEMMs block-scaled (moe_grouped_gemm_mxfp8).  Routing,
 * permutation, combine and bias update as moe_layer_forward.  d and I must
 * be multiples of 256.
 *   w13_sf uint8 [N_r+1, 2I/128, d/128], w2_sf uint8 [N_r+1, d/128, I/128]
 *   ws, ws_bytes scratch of moe_layer_mx_workspace_size(shape) */
typedef struct {
    const uint8_t* w13;
    const uint8_t* w13_sf;
    const uint8_t* w2;
    const uint8_t* w2_sf;
    const uint16_t* router_w;
} MoeWeightsMx;
MOE_API size_t moe_layer_mx_workspace_size(const MoeShape* shape);
MOE_API int moe_layer_forward_mx(const MoeShape* shape, const MoeWeightsMx* weights,
                                 const uint16_t* x, float* bias, const float* logit_offset,
                                 MoeRouting* routing, uint16_t* y, int update_bias, void* ws,
                                 size_t ws_bytes, int* dev_status, void* stream);

/* moe_layer_forward_host_batches: n_batches successive batches of the layer
 * with x and y in HOST memory (pinned), the transfers overlapped with the
 * computation: while batch j runs on `stream`, x of batch j+1 is copied in
 * on one internal copy stream and y of batch j-1 out on another (two device
 * buffers of x and of y alternate in the workspace).  Every output token
 * needs the outputs of every expert, so inside one batch the copies cannot
 * overlap the work; across batches they can.
 *   x_host       bf16 [n_batches, T, d] (pinned for the copies to be
 *                asynchronous);  y_host bf16 [n_batches, T, d] out
 *   bias         updated after each batch when update_bias != 0: batch j
 *                routes with the bias batch j-1 left, exactly as n_batches
 *                calls of moe_layer_forward_host would
 *   routing      holds the last batch's routing when the call completes
 *   ws, ws_bytes scratch of moe_layer_host_batches_workspace_size(shape)
 * Work already queued on `stream` is finished before the first copy starts;
 * `stream` completes after the last copy out: synchronise it before reading
 * y_host.  The two copy streams and the events are created and released by
 * the call.  Errors: those of moe_layer_forward, MOE_ERR_ARG (n_batches <
 * 0).  n_batches = 0 does nothing. */
MOE_API size_t moe_layer_host_batches_workspace_size(const MoeShape* shape);
MOE_API int moe_layer_forward_host_batches(const MoeShape* shape, const MoeWeights* weights,
                                           const uint16_t* x_host, int n_batches, float* bias,
                                           const float* logit_offset, MoeRouting* routing,
                                           uint16_t* y_host, int update_bias, void* ws,
                                           size_t ws_bytes, int* dev_status, void* stream);

/* ====================================================================
 * Backward pass (dx and the router's gradient) of the layer, fp32-scale
 * recipe ("DeepSeek-V3 Technical Report" notes page, section "FP8 mixed
 * precision training": the Dgrad GEMMs take FP8 operands with 1x128 tiles
 * for activation gradients and 128x128 blocks for weights, accumulation in
 * FP32 with per-128-K promotion; section "DeepSeekMoE and
 * auxiliary-loss-free load balancing": the gates are the chosen unbiased
 * affinities normalised, the bias and the top-K choice carry no gradient).
 * The steps for an upstream gradient dy (bf16 [T, d]), with the rows of the
 * forward's permutation (R = T*K + T, the shared expert's row of token t is
 * T*K + t):
 *   moe_combine_backward_quant -> do rows, FP8 1x128 (d)
 *   moe_grouped_gemm_fp8 (do, W2 transposed, n = I, F32)     -> dh
 *   moe_grouped_gemm_fp8 (forward FP8 x rows, W13, n = 2I, F32) -> [a | c]
 *   moe_swiglu_backward_quant -> [da | dc] FP8 1x128 (2I)
 *   moe_grouped_gemm_fp8 ([da|dc], W13 transposed, n = d, F32) -> dx rows
 *   moe_gate_backward, moe_router_backward, moe_dx_combine -> dx, dE.
 * The expert weights' gradients (Wgrad) follow below.
 * ==================================================================== */

/* fp8_transpose_w_128x128: for mats matrices of FP8 codes [rows, cols] with
 * fp32 scales [rows/128, cols/128] (the 128x128 block quantiser's output),
 * write the transposed codes [cols, rows] and scales [cols/128, rows/128].
 * A block keeps its scale, so the transposed matrix holds the same values
 * exactly (no requantisation).  Bit-exact.  rows, cols multiples of 128; q
 * and qt 16-byte aligned.  Errors: MOE_ERR_SHAPE, MOE_ERR_NULL, MOE_ERR_ALIGN,
 * MOE_ERR_CUDA. */
MOE_API int fp8_transpose_w_128x128(const uint8_t* q, const float* scales, int64_t mats,
                                    int64_t rows, int64_t cols, uint8_t* qt, float* scales_t,
                                    int* dev_status, void* stream);

/* moe_combine_backward_quant: the gradient of each expert row's output,
 * do = fp32(gate[t,k] * dy[t]) for the row of (t, k) and do = dy[t] for the
 * shared row of t, quantised like the forward's activations (1x128 tiles
 * along d, scale = amax/448 in fp32, code = E4M3(v * (448/amax))).
 *   dy           bf16 [T, d] device, 16-byte aligned
 *   row_of_pair  int32 [T, K] (the forward's; entries < 0 are skipped)
 *   topk_gate    fp32 [T, K] (the forward's gates)
 *   do_q         uint8 [R, d] out;  do_scales fp32 [d/128, R] out (k-block
 *                major, the grouped GEMM's A-scale layout)
 * Errors: MOE_ERR_SHAPE, MOE_ERR_NULL, MOE_ERR_ALIGN, MOE_ERR_CUDA. */
MOE_API int moe_combine_backward_quant(const MoeShape* shape, const uint16_t* dy,
                                       const int32_t* row_of_pair, const float* topk_gate,
                                       uint8_t* do_q, float* do_scales, int* dev_status,
                                       void* stream);

/* moe_swiglu_backward_quant: for rows of dh (fp32 [rows, I]) and the
 * pre-activations [a | c] (fp32 [rows, 2I]), da = dh c silu'(a) with
 * silu'(a) = sigma(a)(1 + a(1 - sigma(a))) and dc = dh silu(a), in fp32, the
 * row [da | dc] quantised in 1x128 tiles along 2I into q (uint8 [rows, 2I])
 * and q_scales (fp32 [2I/128, rows_total], k-block major).  inter % 128 ==
 * 0; dh, ac, q 16-byte aligned.  Errors: MOE_ERR_SHAPE, MOE_ERR_NULL,
 * MOE_ERR_ALIGN, MOE_ERR_CUDA. */
MOE_API int moe_swiglu_backward_quant(const float* dh, const float* ac, int64_t rows, int inter,
                                      int64_t rows_total, uint8_t* q, float* q_scales,
                                      int* dev_status, void* stream);

/* moe_gate_backward: dgate[t,k] = <dy[t], o[row of (t,k)]> (FP64 sum, stored
 * fp32) and du[t,k], the gradient of the chosen expert's logit:
 * ds_k = (dgate_k - sum_j g_j dgate_j) / S with S = sum of the chosen s,
 * du_k = ds_k s_k (1 - s_k) (FP64, stored fp32).
 *   dy bf16 [T, d]; expert_out fp32 [R, d] (the forward's expert outputs,
 *   ungated); row_of_pair int32 [T, K]; topk_score fp32 [T, K] (from
 *   moe_route_scores); dgate, du fp32 [T, K] out.
 * Errors: MOE_ERR_SHAPE, MOE_ERR_NULL, MOE_ERR_CUDA. */
MOE_API int moe_gate_backward(const MoeShape* shape, const uint16_t* dy, const float* expert_out,
                              const int32_t* row_of_pair, const float* topk_score, float* dgate,
                              float* du, int* dev_status, void* stream);

/* moe_router_backward: the router's two gradients from du (fp32 [T, K]):
 *   dx_router[t] = sum_k du[t,k] E[topk_idx[t,k]]     (fp32 [T, d] out,
 *                  fp32 fused multiply-adds in slot order)
 *   d_router_w[e] = sum over the tokens choosing e of du x[t] (fp32 [N_r, d]
 *                  out; every row written, zero for an unchosen expert),
 *                  summed in a fixed order: the expert's rows (tokens
 *                  ascending) in blocks of 128, each block's rows in order
 *                  into a partial sum, the partials then added in order
 *   x bf16 [T, d]; router_w bf16 [N_r, d]; topk_idx int32 [T, K];
 *   expert_offsets int32 [N_r + 2] and row_of_pair int32 [T, K] (the
 *   forward's permutation); pair_scratch int32 [T*K] out: the
 *   permutation's inverse over the routed rows (pair t*K + k of each row);
 *   ws, ws_bytes scratch of moe_router_backward_workspace_size(shape).
 * Errors: MOE_ERR_SHAPE, MOE_ERR_NULL, MOE_ERR_ALIGN, MOE_ERR_WORKSPACE,
 * MOE_ERR_CUDA; MOE_DEV_BAD_INPUT on dev_status for an expert index out of
 * range. */
MOE_API size_t moe_router_backward_workspace_size(const MoeShape* shape);
MOE_API int moe_router_backward(const MoeShape* shape, const uint16_t* x,
                                const uint16_t* router_w, const float* du,
                                const int32_t* topk_idx, const int32_t* expert_offsets,
                                const int32_t* row_of_pair, int32_t* pair_scratch,
                                float* dx_router, float* d_router_w, void* ws, size_t ws_bytes,
                                int* dev_status, void* stream);

/* moe_dx_combine: dx[t] = dx_rows[shared row of t] + sum_k dx_rows[row of
 * (t,k)] (slot order) + dx_router[t] (NULL: none), fp32 [T, d] out.
 *   dx_rows fp32 [R, d] (the expert rows' input gradients).
 * Errors: MOE_ERR_SHAPE, MOE_ERR_NULL, MOE_ERR_ALIGN, MOE_ERR_CUDA. */
MOE_API int moe_dx_combine(const MoeShape* shape, const float* dx_rows, const float* dx_router,
                           const int32_t* row_of_pair, float* dx, int* dev_status,
                           void* stream);

/* -------------------------------------------------- weight gradients
 * dW13_e [2I, d] = sum over expert e's rows of [da | dc]^T x and
 * dW2_e [d, I] = sum of do^T h (h = silu(a) c), as FP8 GEMMs whose operands
 * are quantised in 128x1 tiles along the rows ("DeepSeek-V3 Technical
 * Report" notes page, section "FP8 mixed precision training": Wgrad in FP8;
 * the pages' request for transposed-operand support).  Each expert's rows,
 * in the forward's permutation order, are cut into K blocks of 128 from its
 * first row; an operand is stored transposed, [features, n_blocks * 128]
 * uint8 codes (a block's 128 codes of a feature contiguous, rows past the
 * expert's end zero) with fp32 scales [n_blocks, features], one per feature
 * and block (amax/448 rule of the 1x128 quantiser).  The value sources:
 * x from the layer input (bf16), do = fp32(gate dy), h and [da | dc] from
 * the recomputed fp32 a and c and dh. */

/* Blocks an operand array must hold for `rows` permutation rows in
 * n_groups groups: ceil(rows/128) + n_groups (-1 for invalid arguments). */
MOE_API int moe_wgrad_max_blocks(int64_t rows, int n_groups);

/* moe_wgrad_layout: from row_offsets (int32 [n_groups + 1], the forward's
 * expert_offsets with the shared expert as the last group) the K-block
 * offsets kb_offsets (int32 [n_groups + 1] out) and the block table blocks
 * (int32 [max_blocks, 2] out: first row, rows; (0, 0) past the last block).
 * One CTA.  More blocks than max_blocks: MOE_DEV_BAD_INPUT on dev_status.
 * Errors: MOE_ERR_SHAPE (n_groups outside [1, 2048], max_blocks < 1),
 * MOE_ERR_NULL, MOE_ERR_CUDA. */
MOE_API int moe_wgrad_layout(int n_groups, const int32_t* row_offsets, int max_blocks,
                             int32_t* kb_offsets, int32_t* blocks, int* dev_status, void* stream);

/* The 128x1 quantisers (blocks / n_blocks: the layout's table and its
 * length, which is also the K extent of the output arrays):
 *   moe_wgrad_quant_x:   x bf16 [T, d] -> xt [d, n_blocks*128], scales
 *                        [n_blocks, d]; row r takes the token of its pair
 *                        (pair_of_row, the permutation's inverse over the
 *                        T*K routed rows, as moe_router_backward leaves it in
 *                        pair_scratch), shared row T*K + t token t;
 *   moe_wgrad_quant_do:  the same with fp32(topk_gate[pair] * dy) (dy on the
 *                        shared rows) -> dot [d, ...];
 *   moe_wgrad_quant_h:   ac fp32 [rows, 2I] -> ht [I, ...] of
 *                        h = a / (1 + e^-a) * c;
 *   moe_wgrad_quant_dac: dh fp32 [rows, I], ac -> dact [2I, ...] of
 *                        [da | dc] as moe_swiglu_backward_quant forms them.
 * Output codes 16-byte aligned.  Errors: MOE_ERR_SHAPE, MOE_ERR_NULL,
 * MOE_ERR_ALIGN, MOE_ERR_CUDA. */
MOE_API int moe_wgrad_quant_x(const MoeShape* shape, const uint16_t* x,
                              const int32_t* pair_of_row, const int32_t* blocks, int n_blocks,
                              uint8_t* xt, float* xt_scales, int* dev_status, void* stream);
MOE_API int moe_wgrad_quant_do(const MoeShape* shape, const uint16_t* dy, const float* topk_gate,
                               const int32_t* pair_of_row, const int32_t* blocks, int n_blocks,
                               uint8_t* dot, float* dot_scales, int* dev_status, void* stream);
MOE_API int moe_wgrad_quant_h(const float* ac, int inter, const int32_t* blocks, int n_blocks,
                              uint8_t* ht, float* ht_scales, int* dev_status, void* stream);
MOE_API int moe_wgrad_quant_dac(const float* dh, const float* ac, int inter,
                                const int32_t* blocks, int n_blocks, uint8_t* dact,
                                float* dact_scales, int* dev_status, void* stream);

/* moe_grouped_gemm_wgrad: out[g] (fp32 [m, n], groups back to back) =
 * sum over the K blocks kb in [kb_offsets[g], kb_offsets[g+1]) of
 * a_scales[kb, i] b_scales[kb, j] sum_{k in kb} A[i, k] B[j, k], the
 * products exact on the tensor cores, each K block promoted into an FP32
 * accumulator with its two scales; a group with no K blocks gets zeros.
 *   a_t uint8 [m, nkb_total*128] (E4M3), a_scales fp32 [nkb_total, m];
 *   b_t uint8 [n, nkb_total*128], b_scales fp32 [nkb_total, n];
 *   kb_offsets int32 [n_groups + 1], non-decreasing, within [0, nkb_total]
 *   (else MOE_DEV_BAD_INPUT on dev_status and nothing is computed).
 * m % 128 == 0, n % 256 == 0, pointers 16-byte aligned.  Errors:
 * MOE_ERR_SHAPE, MOE_ERR_NULL, MOE_ERR_ALIGN, MOE_ERR_DEVICE, MOE_ERR_CUDA;
 * MOE_DEV_TIMEOUT as the forward GEMM. */
MOE_API int moe_grouped_gemm_wgrad(int n_groups, const int32_t* kb_offsets, int nkb_total,
                                   const uint8_t* a_t, const float* a_scales, int m,
                                   const uint8_t* b_t, const float* b_scales, int n, float* out,
                                   int* dev_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOEFP8_H */
