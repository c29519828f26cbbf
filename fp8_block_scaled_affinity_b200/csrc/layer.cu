// Whole MoE layer forward on one stream, workspace layout, status helpers.
// The order of stages follows the MoE block of "DeepSeek-V3 Technical
// Report" (notes page): gating (section "DeepSeekMoE and auxiliary-loss-free
// load balancing"), FP8 quantisation of the dispatched activations, dispatch,
// expert MLP in FP8 (section "FP8 mixed precision training"), combine
// (section "DualPipe"), and the bias update from the batch's expert load.
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "common.cuh"

namespace moe {

int sm_count() {
    static int counts[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (counts[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        counts[dev] = n;
    }
    return counts[dev];
}

bool device_accessible(const void* p) {
    if (!p) return true;
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        (void)cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged ||
           a.type == cudaMemoryTypeHost;
}

uint64_t wait_limit_ns() {
    const char* env = getenv("MOEFP8_WAIT_LIMIT_NS");
    if (!env || !*env) return kWaitLimitNs;
    char* end = nullptr;
    const unsigned long long v = strtoull(env, &end, 10);
    if (end == env || v == 0) return kWaitLimitNs;
    return v < 1000ull ? 1000ull : v;  // at least 1 us
}

int fault_injection() {
    const char* env = getenv("MOEFP8_FAULT");
    if (env && strcmp(env, "gemm_producer") == 0) return kFaultGemmProducer;
    return kFaultNone;
}

namespace {

// Workspace of the layer: every piece starts on a 256-byte boundary.
struct LayerWs {
    uint8_t* xq_perm;  // [R, d]      R = T*K + T
    float* xs_perm;    // [d/128, R]
    uint8_t* hq;       // [R, I]
    float* hs;         // [I/128, R]
    float* o;          // [R, d]
    void* route_ws;
    void* perm_ws;
    uint16_t* x_dev;   // host variants only: [T, d] (two buffers for batches)
    uint16_t* y_dev;   // host variants only: [T, d] (two buffers for batches)
    uint16_t* x_dev2;
    uint16_t* y_dev2;
    size_t bytes;
};

// host_io: 0 device buffers only, 1 one x and one y buffer, 2 two of each
LayerWs carve(const MoeShape* s, void* base, int host_io) {
    LayerWs w{};
    const size_t T = s->T, d = s->d, I = s->inter;
    const size_t R = T * s->topk + T;
    uintptr_t p = reinterpret_cast<uintptr_t>(base);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off = align_up(off + bytes, 256);
        return reinterpret_cast<void*>(p + at);
    };
    w.xq_perm = static_cast<uint8_t*>(take(R * d));
    w.xs_perm = static_cast<float*>(take((d / 128) * R * 4));
    w.hq = static_cast<uint8_t*>(take(R * I));
    w.hs = static_cast<float*>(take((I / 128) * R * 4));
    w.o = static_cast<float*>(take(R * d * 4));
    w.route_ws = take(moe_route_workspace_size(s));
    w.perm_ws = take(moe_permute_workspace_size(s));
    if (host_io >= 1) {
        w.x_dev = static_cast<uint16_t*>(take(T * d * 2));
        w.y_dev = static_cast<uint16_t*>(take(T * d * 2));
    }
    if (host_io >= 2) {
        w.x_dev2 = static_cast<uint16_t*>(take(T * d * 2));
        w.y_dev2 = static_cast<uint16_t*>(take(T * d * 2));
    }
    w.bytes = off;
    return w;
}

// x_consumed (nullable) is recorded on `stream` once x has been read for
// the last time (after the quantise + permute pass).
int run_layer(const MoeShape* s, const MoeWeights* wt, const uint16_t* x, float* bias,
              const float* logit_offset, MoeRouting* rt, uint16_t* y, int update_bias,
              const LayerWs& w, int* dev_status, void* stream,
              cudaEvent_t x_consumed = nullptr) {
    const int T = s->T, d = s->d, I = s->inter, N = s->n_routed, K = s->topk;
    const int R = T * K + T;
    int rc = moe_route(s, x, wt->router_w, bias, logit_offset, rt->topk_idx, rt->topk_gate,
                       rt->expert_counts, w.route_ws, moe_route_workspace_size(s), dev_status,
                       stream);
    if (rc != MOE_OK) return rc;
    rc = moe_quant_permute(s, x, rt->topk_idx, rt->expert_counts, w.xq_perm, w.xs_perm,
                           rt->expert_offsets, rt->row_of_pair, w.perm_ws,
                           moe_permute_workspace_size(s), dev_status, stream);
    if (rc != MOE_OK) return rc;
    if (x_consumed && cudaEventRecord(x_consumed, as_stream(stream)) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (T > 0) {
        rc = moe_grouped_gemm_fp8(N + 1, rt->expert_offsets, R, w.xq_perm, w.xs_perm, d,
                                  wt->w13, wt->w13_scales, 2 * I, MOE_EPI_SWIGLU_QUANT, w.hq,
                                  w.hs, dev_status, stream);
        if (rc != MOE_OK) return rc;
        rc = moe_grouped_gemm_fp8(N + 1, rt->expert_offsets, R, w.hq, w.hs, I, wt->w2,
                                  wt->w2_scales, d, MOE_EPI_F32, w.o, nullptr, dev_status, stream);
        if (rc != MOE_OK) return rc;
        rc = moe_combine(s, w.o, rt->expert_offsets, rt->row_of_pair, rt->topk_gate, y,
                         dev_status, stream);
        if (rc != MOE_OK) return rc;
    }
    if (update_bias) rc = moe_update_bias(s, rt->expert_counts, bias, dev_status, stream);
    return rc;
}

int check_layer_args(const MoeShape* s, const MoeWeights* wt, float* bias, MoeRouting* rt,
                     void* ws) {
    int rc = validate_shape(s);
    if (rc != MOE_OK) return rc;
    if (!wt || !rt || !bias || !ws) return MOE_ERR_NULL;
    if (!wt->w13 || !wt->w13_scales || !wt->w2 || !wt->w2_scales || !wt->router_w)
        return MOE_ERR_NULL;
    if (!rt->expert_counts || !rt->expert_offsets) return MOE_ERR_NULL;
    if (s->T > 0 && (!rt->topk_idx || !rt->topk_gate || !rt->row_of_pair)) return MOE_ERR_NULL;
    if (int64_t(s->T) * (s->topk + 1) * s->d > (int64_t(1) << 40)) return MOE_ERR_SHAPE;
    return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" MOE_API int moe_version(void) { return 100; }

extern "C" MOE_API const char* moe_status_string(int status) {
    switch (status) {
        case MOE_OK: return "ok";
        case MOE_ERR_NULL: return "a required pointer is NULL";
        case MOE_ERR_SHAPE: return "unsupported size";
        case MOE_ERR_ROUTE: return "inconsistent routing shape";
        case MOE_ERR_CUDA: return "CUDA launch or runtime call failed";
        case MOE_ERR_ALIGN: return "pointer not 16-byte aligned";
        case MOE_ERR_WORKSPACE: return "workspace missing or too small";
        case MOE_ERR_ARG: return "invalid argument";
        case MOE_ERR_DEVICE: return "device is not sm_100 (B200)";
        case MOE_ERR_STATIC_LIMIT:
            return "shape exceeds the fixed scratch of the no-allocation entry point";
        default: return "unknown status";
    }
}

extern "C" MOE_API int moe_read_status(const int* dev_status, int* host_status, void* stream) {
    if (!dev_status || !host_status) return MOE_ERR_NULL;
    cudaStream_t st = as_stream(stream);
    if (cudaMemcpyAsync(host_status, dev_status, sizeof(int), cudaMemcpyDeviceToHost, st) !=
            cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

extern "C" MOE_API size_t moe_layer_workspace_size(const MoeShape* shape) {
    if (validate_shape(shape) != MOE_OK) return 0;
    return carve(shape, nullptr, 0).bytes;
}

extern "C" MOE_API size_t moe_layer_host_workspace_size(const MoeShape* shape) {
    if (validate_shape(shape) != MOE_OK) return 0;
    return carve(shape, nullptr, 1).bytes;
}

extern "C" MOE_API size_t moe_layer_host_batches_workspace_size(const MoeShape* shape) {
    if (validate_shape(shape) != MOE_OK) return 0;
    return carve(shape, nullptr, 2).bytes;
}

extern "C" MOE_API int moe_layer_forward(const MoeShape* shape, const MoeWeights* weights,
                                         const uint16_t* x, float* bias,
                                         const float* logit_offset, MoeRouting* routing,
                                         uint16_t* y, int update_bias, void* ws, size_t ws_bytes,
                                         int* dev_status, void* stream) {
    int rc = check_layer_args(shape, weights, bias, routing, ws);
    if (rc != MOE_OK) return rc;
    if (shape->T > 0 && (!x || !y)) return MOE_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(ws) & 255) return MOE_ERR_ALIGN;
    const LayerWs w = carve(shape, ws, 0);
    if (ws_bytes < w.bytes) return MOE_ERR_WORKSPACE;
    return run_layer(shape, weights, x, bias, logit_offset, routing, y, update_bias, w,
                     dev_status, stream);
}

extern "C" MOE_API int moe_layer_forward_host(const MoeShape* shape, const MoeWeights* weights,
                                              const uint16_t* x_host, float* bias,
                                              const float* logit_offset, MoeRouting* routing,
                                              uint16_t* y_host, int update_bias, void* ws,
                                              size_t ws_bytes, int* dev_status, void* stream) {
    int rc = check_layer_args(shape, weights, bias, routing, ws);
    if (rc != MOE_OK) return rc;
    if (shape->T > 0 && (!x_host || !y_host)) return MOE_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(ws) & 255) return MOE_ERR_ALIGN;
    const LayerWs w = carve(shape, ws, 1);
    if (ws_bytes < w.bytes) return MOE_ERR_WORKSPACE;
    const size_t xbytes = size_t(shape->T) * shape->d * sizeof(uint16_t);
    cudaStream_t st = as_stream(stream);
    if (xbytes && cudaMemcpyAsync(w.x_dev, x_host, xbytes, cudaMemcpyHostToDevice, st) !=
                      cudaSuccess)
        return MOE_ERR_CUDA;
    rc = run_layer(shape, weights, w.x_dev, bias, logit_offset, routing, w.y_dev, update_bias, w,
                   dev_status, stream);
    if (rc != MOE_OK) return rc;
    if (xbytes && cudaMemcpyAsync(y_host, w.y_dev, xbytes, cudaMemcpyDeviceToHost, st) !=
                      cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

// Several batches from and to host memory, transfers overlapped with compute:
// the host-to-device copy of batch j+1 runs on one copy stream and the
// device-to-host copy of batch j-1 on another while batch j is computed on
// `stream`; two device buffers of x and of y alternate.  Batches run in
// order and share the bias (each routes with the bias the previous one left
// when update_bias is set), exactly as n_batches calls of
// moe_layer_forward_host would.
namespace moe {
namespace {

struct BatchSync {
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t start = nullptr, done = nullptr;
    cudaEvent_t x_ready[2] = {nullptr, nullptr};  // x of the batch in buffer b copied
    cudaEvent_t x_free[2] = {nullptr, nullptr};   // buffer b's x read for the last time
    cudaEvent_t y_ready[2] = {nullptr, nullptr};  // y of the batch in buffer b computed
    cudaEvent_t y_free[2] = {nullptr, nullptr};   // buffer b's y copied out
    bool ok = true;
    BatchSync() {
        ok = cudaStreamCreateWithFlags(&h2d, cudaStreamNonBlocking) == cudaSuccess &&
             cudaStreamCreateWithFlags(&d2h, cudaStreamNonBlocking) == cudaSuccess &&
             cudaEventCreateWithFlags(&start, cudaEventDisableTiming) == cudaSuccess &&
             cudaEventCreateWithFlags(&done, cudaEventDisableTiming) == cudaSuccess;
        for (int b = 0; ok && b < 2; ++b)
            ok = cudaEventCreateWithFlags(&x_ready[b], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&x_free[b], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&y_ready[b], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&y_free[b], cudaEventDisableTiming) == cudaSuccess;
    }
    // Destroying a stream or an event with work pending is allowed: the
    // resources are released once that work has completed.
    ~BatchSync() {
        for (cudaEvent_t e : {start, done, x_ready[0], x_ready[1], x_free[0], x_free[1],
                              y_ready[0], y_ready[1], y_free[0], y_free[1]})
            if (e) cudaEventDestroy(e);
        if (h2d) cudaStreamDestroy(h2d);
        if (d2h) cudaStreamDestroy(d2h);
    }
};

}  // namespace
}  // namespace moe

extern "C" MOE_API int moe_layer_forward_host_batches(
    const MoeShape* shape, const MoeWeights* weights, const uint16_t* x_host, int n_batches,
    float* bias, const float* logit_offset, MoeRouting* routing, uint16_t* y_host,
    int update_bias, void* ws, size_t ws_bytes, int* dev_status, void* stream) {
    int rc = check_layer_args(shape, weights, bias, routing, ws);
    if (rc != MOE_OK) return rc;
    if (n_batches < 0) return MOE_ERR_ARG;
    if (n_batches == 0) return MOE_OK;
    if (shape->T > 0 && (!x_host || !y_host)) return MOE_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(ws) & 255) return MOE_ERR_ALIGN;
    const LayerWs w = carve(shape, ws, 2);
    if (ws_bytes < w.bytes) return MOE_ERR_WORKSPACE;
    const size_t xbytes = size_t(shape->T) * shape->d * sizeof(uint16_t);
    const size_t xelems = size_t(shape->T) * shape->d;
    cudaStream_t st = as_stream(stream);
    BatchSync sy;
    if (!sy.ok) return MOE_ERR_CUDA;
    uint16_t* xb[2] = {w.x_dev, w.x_dev2};
    uint16_t* yb[2] = {w.y_dev, w.y_dev2};
    // the copy streams start after the work already queued on `stream`
    if (cudaEventRecord(sy.start, st) != cudaSuccess ||
        cudaStreamWaitEvent(sy.h2d, sy.start, 0) != cudaSuccess ||
        cudaStreamWaitEvent(sy.d2h, sy.start, 0) != cudaSuccess)
        return MOE_ERR_CUDA;
    auto h2d = [&](int j) -> int {
        const int b = j & 1;
        if (j >= 2 && cudaStreamWaitEvent(sy.h2d, sy.x_free[b], 0) != cudaSuccess)
            return MOE_ERR_CUDA;
        if (xbytes && cudaMemcpyAsync(xb[b], x_host + size_t(j) * xelems, xbytes,
                                      cudaMemcpyHostToDevice, sy.h2d) != cudaSuccess)
            return MOE_ERR_CUDA;
        return cudaEventRecord(sy.x_ready[b], sy.h2d) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
    };
    if ((rc = h2d(0)) != MOE_OK) return rc;
    for (int j = 0; j < n_batches; ++j) {
        const int b = j & 1;
        if (j + 1 < n_batches && (rc = h2d(j + 1)) != MOE_OK) return rc;
        if (cudaStreamWaitEvent(st, sy.x_ready[b], 0) != cudaSuccess) return MOE_ERR_CUDA;
        // y buffer b was last used by batch j-2: its copy out must be done
        if (j >= 2 && cudaStreamWaitEvent(st, sy.y_free[b], 0) != cudaSuccess)
            return MOE_ERR_CUDA;
        rc = run_layer(shape, weights, xb[b], bias, logit_offset, routing, yb[b], update_bias, w,
                       dev_status, stream, sy.x_free[b]);
        if (rc != MOE_OK) return rc;
        if (cudaEventRecord(sy.y_ready[b], st) != cudaSuccess ||
            cudaStreamWaitEvent(sy.d2h, sy.y_ready[b], 0) != cudaSuccess)
            return MOE_ERR_CUDA;
        if (xbytes && cudaMemcpyAsync(y_host + size_t(j) * xelems, yb[b], xbytes,
                                      cudaMemcpyDeviceToHost, sy.d2h) != cudaSuccess)
            return MOE_ERR_CUDA;
        if (cudaEventRecord(sy.y_free[b], sy.d2h) != cudaSuccess) return MOE_ERR_CUDA;
    }
    // `stream` completes only after the last copy out
    if (cudaEventRecord(sy.done, sy.d2h) != cudaSuccess ||
        cudaStreamWaitEvent(st, sy.done, 0) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

// The layer with the power-of-two scale option: every FP8 operand (x, the
// expert weights, h) carries UE8M0 scale bytes and both expert GEMMs run as
// block-scaled tensor-core MMAs (moe_grouped_gemm_mxfp8).  Routing, the
// permutation, the combine and the bias update are those of
// moe_layer_forward.
extern "C" MOE_API size_t moe_layer_mx_workspace_size(const MoeShape* shape) {
    return moe_layer_workspace_size(shape);
}

extern "C" MOE_API int moe_layer_forward_mx(const MoeShape* shape, const MoeWeightsMx* wt,
                                            const uint16_t* x, float* bias,
                                            const float* logit_offset, MoeRouting* rt,
                                            uint16_t* y, int update_bias, void* ws,
                                            size_t ws_bytes, int* dev_status, void* stream) {
    int rc = validate_shape(shape);
    if (rc != MOE_OK) return rc;
    if (!wt || !rt || !bias || !ws) return MOE_ERR_NULL;
    if (!wt->w13 || !wt->w13_sf || !wt->w2 || !wt->w2_sf || !wt->router_w) return MOE_ERR_NULL;
    if (!rt->expert_counts || !rt->expert_offsets) return MOE_ERR_NULL;
    if (shape->T > 0 && (!rt->topk_idx || !rt->topk_gate || !rt->row_of_pair || !x || !y))
        return MOE_ERR_NULL;
    if (shape->d % 256 || shape->inter % 256) return MOE_ERR_SHAPE;  // 256-column tiles
    if (reinterpret_cast<uintptr_t>(ws) & 255) return MOE_ERR_ALIGN;
    const LayerWs w = carve(shape, ws, 0);
    if (ws_bytes < w.bytes) return MOE_ERR_WORKSPACE;
    const int T = shape->T, d = shape->d, I = shape->inter, N = shape->n_routed, K = shape->topk;
    const int R = T * K + T;
    // the fp32 scale areas of the workspace hold the scale bytes here
    uint8_t* xsf = reinterpret_cast<uint8_t*>(w.xs_perm);
    uint8_t* hsf = reinterpret_cast<uint8_t*>(w.hs);
    rc = moe_route(shape, x, wt->router_w, bias, logit_offset, rt->topk_idx, rt->topk_gate,
                   rt->expert_counts, w.route_ws, moe_route_workspace_size(shape), dev_status,
                   stream);
    if (rc != MOE_OK) return rc;
    rc = moe_quant_permute_ue8m0(shape, x, rt->topk_idx, rt->expert_counts, w.xq_perm, xsf,
                                 rt->expert_offsets, rt->row_of_pair, w.perm_ws,
                                 moe_permute_workspace_size(shape), dev_status, stream);
    if (rc != MOE_OK) return rc;
    if (T > 0) {
        rc = moe_grouped_gemm_mxfp8(N + 1, rt->expert_offsets, R, w.xq_perm, xsf, d, wt->w13,
                                    wt->w13_sf, 2 * I, MOE_EPI_SWIGLU_QUANT, w.hq, hsf,
                                    dev_status, stream);
        if (rc != MOE_OK) return rc;
        rc = moe_grouped_gemm_mxfp8(N + 1, rt->expert_offsets, R, w.hq, hsf, I, wt->w2,
                                    wt->w2_sf, d, MOE_EPI_F32, w.o, nullptr, dev_status, stream);
        if (rc != MOE_OK) return rc;
        rc = moe_combine(shape, w.o, rt->expert_offsets, rt->row_of_pair, rt->topk_gate, y,
                         dev_status, stream);
        if (rc != MOE_OK) return rc;
    }
    if (update_bias) rc = moe_update_bias(shape, rt->expert_counts, bias, dev_status, stream);
    return rc;
}
