// Whole MoE layer forward on one stream, workspace layout, status helpers.
// The order of stages follows the MoE block of "DeepSeek-V3 Technical
// Report" (notes page): gating (section "DeepSeekMoE and auxiliary-loss-free
// load balancing"), FP8 quantisation of the dispatched activations, dispatch,
// expert MLP in FP8 (section "FP8 mixed precision training"), combine
// (section "DualPipe"), and the bias update from the batch's expert load.
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
    uint16_t* x_dev;   // host variant only: [T, d]
    uint16_t* y_dev;   // host variant only: [T, d]
    size_t bytes;
};

LayerWs carve(const MoeShape* s, void* base, bool host_io) {
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
    if (host_io) {
        w.x_dev = static_cast<uint16_t*>(take(T * d * 2));
        w.y_dev = static_cast<uint16_t*>(take(T * d * 2));
    }
    w.bytes = off;
    return w;
}

int run_layer(const MoeShape* s, const MoeWeights* wt, const uint16_t* x, float* bias,
              const float* logit_offset, MoeRouting* rt, uint16_t* y, int update_bias,
              const LayerWs& w, int* dev_status, void* stream) {
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
    return carve(shape, nullptr, false).bytes;
}

extern "C" MOE_API size_t moe_layer_host_workspace_size(const MoeShape* shape) {
    if (validate_shape(shape) != MOE_OK) return 0;
    return carve(shape, nullptr, true).bytes;
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
    const LayerWs w = carve(shape, ws, false);
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
    const LayerWs w = carve(shape, ws, true);
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
