"""B200-native DeepSeekMoE layer forward with FP8 block scaling.

The compute lives in libmoefp8.so (hand-written sm_100a CUDA kernels behind a
C ABI, declared in include/moefp8.h).  This package is the thin Python side:
the ctypes binding with the C names (``_lib``) and ``MoeLayer``, which owns
the device buffers of one layer (allocated with torch) and calls the library.
There is no CPU or PyTorch fallback: if the library is missing, loading it
raises.
"""
from __future__ import annotations

from typing import Optional

from ._lib import (MOE_DEV_TIMEOUT, MOE_EPI_BF16, MOE_EPI_F32, MOE_EPI_SWIGLU_QUANT,  # noqa: F401
                   MoeError, MoeRouting, MoeShape, MoeWeights, fp8_quant_act_1x128,
                   fp8_quant_w_128x128, lib, make_routing, make_shape, make_weights,
                   moe_combine, moe_grouped_gemm_form, moe_grouped_gemm_fp8,
                   moe_layer_forward, moe_layer_forward_host_batches,
                   moe_layer_forward_host, moe_layer_host_batches_workspace_size,
                   moe_layer_host_workspace_size,
                   moe_layer_workspace_size, moe_permute, moe_permute_workspace_size, moe_quant_permute,
                   moe_read_status, moe_route, moe_route_workspace_size, moe_update_bias,
                   moe_version, status_string, fp8_quant_act_1x128_ue8m0,
                   fp8_quant_w_128x128_ue8m0, moe_grouped_gemm_mxfp8,
                   moe_grouped_gemm_fp8_indexed, moe_plan_redundant_experts, moe_split_groups,
                   MoeWeightsMx, make_weights_mx, moe_layer_forward_mx,
                   moe_layer_mx_workspace_size, moe_quant_permute_ue8m0,
                   moe_ep_row_bytes, moe_ep_workspace_size, moe_ep_dispatch_plan, moe_ep_pack,
                   moe_ep_local_permute, moe_ep_partial_combine, moe_ep_final_combine,
                   moe_route_scores, fp8_transpose_w_128x128, moe_combine_backward_quant,
                   moe_swiglu_backward_quant, moe_gate_backward, moe_router_backward,
                   moe_router_backward_workspace_size,
                   moe_dx_combine, moe_wgrad_max_blocks, moe_wgrad_layout, moe_wgrad_quant_x,
                   moe_wgrad_quant_do, moe_wgrad_quant_h, moe_wgrad_quant_dac,
                   moe_grouped_gemm_wgrad)

__all__ = ["MoeLayer", "MoeShape", "MoeError", "lib", "make_shape", "moe_version"]


class MoeLayer:
    """Device state of one MoE layer: FP8 expert weights, router weights,
    the balancing bias and the workspace.

    shape: a MoeShape (see make_shape).  router_w: bf16 [N_r, d] on the GPU.
    bias: fp32 [N_r] on the GPU (updated in place by forward(update_bias=True)).
    """

    def __init__(self, shape: MoeShape, router_w, bias, device=None, host_io=False,
                 scales: str = "fp32"):
        """scales: "fp32" (the pages' recipe: FP32 scales, per-128-K promotion)
        or "ue8m0" (power-of-two scales, block-scaled tensor-core GEMMs)."""
        import torch
        if scales not in ("fp32", "ue8m0"):
            raise ValueError("scales must be 'fp32' or 'ue8m0'")
        if scales == "ue8m0" and host_io:
            raise ValueError("host-buffer calls use the fp32-scale layer")
        self.scales = scales
        self.shape = shape
        dev = torch.device(device) if device is not None else router_w.device
        self.device = dev
        N, d, I = shape.n_routed, shape.d, shape.inter
        E = N + 1
        self.router_w = router_w
        self.bias = bias
        u8 = torch.uint8
        self.w13 = torch.empty((E, 2 * I, d), dtype=u8, device=dev)
        sdt = torch.float32 if scales == "fp32" else u8  # UE8M0 bytes for "ue8m0"
        self.w13_scales = torch.empty((E, 2 * I // 128, d // 128), dtype=sdt, device=dev)
        self.w2 = torch.empty((E, d, I), dtype=u8, device=dev)
        self.w2_scales = torch.empty((E, d // 128, I // 128), dtype=sdt, device=dev)
        T, K = shape.T, shape.topk
        i32 = torch.int32
        self.topk_idx = torch.empty((T, K), dtype=i32, device=dev)
        self.topk_gate = torch.empty((T, K), dtype=torch.float32, device=dev)
        self.expert_counts = torch.empty((N,), dtype=i32, device=dev)
        self.expert_offsets = torch.empty((N + 2,), dtype=i32, device=dev)
        self.row_of_pair = torch.empty((T, K), dtype=i32, device=dev)
        self.dev_status = torch.zeros((1,), dtype=i32, device=dev)
        # host_io: False (device x / y), True (forward_host), "batches"
        # (forward_host_batches as well)
        ws_bytes = (moe_layer_host_batches_workspace_size(shape) if host_io == "batches"
                    else moe_layer_host_workspace_size(shape) if host_io
                    else moe_layer_workspace_size(shape))
        self.ws = torch.empty((max(ws_bytes, 256),), dtype=u8, device=dev)
        self._weights = None
        self._transposed = None
        self._train = None
        self._routing = make_routing(self.topk_idx, self.topk_gate, self.expert_counts,
                                     self.expert_offsets, self.row_of_pair)

    def set_expert(self, e: int, w1, w3, w2, stream=None) -> None:
        """Quantise expert e's bf16 weights (W1, W3: [I, d]; W2: [d, I]) into
        the layer's FP8 buffers with 128x128 blocks.  e = N_r is the shared
        expert."""
        I = self.shape.inter
        quant = fp8_quant_w_128x128 if self.scales == "fp32" else fp8_quant_w_128x128_ue8m0
        quant(w1, self.w13[e, :I], self.w13_scales[e, :I // 128], stream=stream)
        quant(w3, self.w13[e, I:], self.w13_scales[e, I // 128:], stream=stream)
        quant(w2, self.w2[e], self.w2_scales[e], stream=stream)
        self._weights = None
        self._transposed = None

    def weights(self):
        if self._weights is None:
            mk = make_weights if self.scales == "fp32" else make_weights_mx
            self._weights = mk(self.w13, self.w13_scales, self.w2, self.w2_scales, self.router_w)
        return self._weights

    def forward(self, x, y=None, update_bias: bool = False, logit_offset=None, stream=None):
        """y = MoE(x) for bf16 x [T, d] on the GPU; returns y (bf16 [T, d])."""
        import torch
        if y is None:
            y = torch.empty_like(x)
        fwd = moe_layer_forward if self.scales == "fp32" else moe_layer_forward_mx
        fwd(self.shape, self.weights(), x, self.bias, logit_offset, self._routing, y,
            update_bias, self.ws, self.dev_status, stream)
        return y

    def forward_host(self, x_host, y_host, update_bias: bool = False, logit_offset=None,
                     stream=None):
        """The same with x and y in (pinned) host memory; the copies run on
        `stream` inside the call.  Synchronise the stream before reading y."""
        moe_layer_forward_host(self.shape, self.weights(), x_host, self.bias, logit_offset,
                               self._routing, y_host, update_bias, self.ws, self.dev_status,
                               stream)

    def forward_host_batches(self, x_host, y_host, update_bias: bool = False,
                             logit_offset=None, stream=None):
        """Batches x_host[j] (pinned bf16 [n, T, d]) -> y_host[j], the copies
        of neighbouring batches overlapped with the computation (the layer
        must be built with host_io="batches").  Synchronise the stream before
        reading y_host."""
        moe_layer_forward_host_batches(self.shape, self.weights(), x_host, x_host.shape[0],
                                       self.bias, logit_offset, self._routing, y_host,
                                       update_bias, self.ws, self.dev_status, stream)

    # ------------------------------------------------------------ training
    def _train_buffers(self):
        import torch
        if self._train is None:
            sh, dev = self.shape, self.device
            T, d, I, K = sh.T, sh.d, sh.inter, sh.topk
            R = T * K + T
            u8, f32, i32 = torch.uint8, torch.float32, torch.int32
            self._train = {
                "score": torch.empty((T, K), dtype=f32, device=dev),
                "route_ws": torch.empty((max(moe_route_workspace_size(sh), 256),), dtype=u8,
                                        device=dev),
                "perm_ws": torch.empty((max(moe_permute_workspace_size(sh), 256),), dtype=u8,
                                       device=dev),
                "xq": torch.empty((R, d), dtype=u8, device=dev),
                "xs": torch.empty((d // 128, R), dtype=f32, device=dev),
                "hq": torch.empty((R, I), dtype=u8, device=dev),
                "hs": torch.empty((I // 128, R), dtype=f32, device=dev),
                "o": torch.empty((R, d), dtype=f32, device=dev),
                "x": None,
            }
        return self._train

    def forward_train(self, x, y=None, update_bias: bool = False, logit_offset=None,
                      stream=None):
        """The forward pass (fp32-scale recipe) through the stage entry points,
        keeping what backward() needs: the chosen affinities, the permuted FP8
        rows and the expert outputs.  y equals forward()'s bit for bit; x
        must stay unchanged until backward() has run."""
        import torch
        if self.scales != "fp32":
            raise ValueError("the backward pass uses the fp32-scale layer")
        sh, b = self.shape, self._train_buffers()
        N, d, I, K, T = sh.n_routed, sh.d, sh.inter, sh.topk, sh.T
        R = T * K + T
        if y is None:
            y = torch.empty_like(x)
        st = self.dev_status
        moe_route_scores(sh, x, self.router_w, self.bias, logit_offset, self.topk_idx,
                         self.topk_gate, b["score"], self.expert_counts, b["route_ws"], st,
                         stream)
        moe_quant_permute(sh, x, self.topk_idx, self.expert_counts, b["xq"], b["xs"],
                          self.expert_offsets, self.row_of_pair, b["perm_ws"], st, stream)
        moe_grouped_gemm_fp8(N + 1, self.expert_offsets, R, b["xq"], b["xs"], d, self.w13,
                             self.w13_scales, 2 * I, MOE_EPI_SWIGLU_QUANT, b["hq"], b["hs"], st,
                             stream)
        moe_grouped_gemm_fp8(N + 1, self.expert_offsets, R, b["hq"], b["hs"], I, self.w2,
                             self.w2_scales, d, MOE_EPI_F32, b["o"], None, st, stream)
        moe_combine(sh, b["o"], self.expert_offsets, self.row_of_pair, self.topk_gate, y, st,
                    stream)
        if update_bias:
            moe_update_bias(sh, self.expert_counts, self.bias, st, stream)
        b["x"] = x
        return y

    def _transposed_weights(self, stream=None):
        """W2 and W13 with rows and columns swapped (the Dgrad GEMMs' B
        operands): the same FP8 codes and 128x128 scales, moved."""
        import torch
        if self._transposed is None:
            sh, dev = self.shape, self.device
            E, d, I = sh.n_routed + 1, sh.d, sh.inter
            u8, f32 = torch.uint8, torch.float32
            w2t = torch.empty((E, I, d), dtype=u8, device=dev)
            w2t_s = torch.empty((E, I // 128, d // 128), dtype=f32, device=dev)
            w13t = torch.empty((E, d, 2 * I), dtype=u8, device=dev)
            w13t_s = torch.empty((E, d // 128, 2 * I // 128), dtype=f32, device=dev)
            fp8_transpose_w_128x128(self.w2, self.w2_scales, w2t, w2t_s, self.dev_status, stream)
            fp8_transpose_w_128x128(self.w13, self.w13_scales, w13t, w13t_s, self.dev_status,
                                    stream)
            self._transposed = (w2t, w2t_s, w13t, w13t_s)
        return self._transposed

    def backward(self, dy, stream=None, marks=None, wgrad: bool = False):
        """Gradients of the last forward_train() for the upstream gradient dy
        (bf16 [T, d]): returns (dx fp32 [T, d], d_router_w fp32 [N_r, d]), and
        with wgrad=True also the expert weights' gradients dW13 (fp32
        [N_r + 1, 2I, d], W1 rows then W3 rows) and dW2 (fp32 [N_r + 1, d, I]),
        the shared expert last.

        Dgrad through the experts with FP8 operands (the gate-scaled output
        gradient and [da | dc] quantised in 1x128 tiles, the weights' own
        128x128 blocks transposed), a and c recomputed from the forward's FP8
        rows; the gate and router gradients in high precision.  The top-K
        choice and the bias carry no gradient.  The weight gradients are FP8
        GEMMs over each expert's rows with both operands quantised in 128x1
        tiles along the rows (x from the layer input, do = gate dy, h and
        [da | dc] from the recomputed fp32 a, c).

        marks: a list, or None; given a list, a timing CUDA event recorded on
        the stream after each stage is appended as (stage name, event), with
        ("start", event) first."""
        import torch
        b = self._train
        if b is None or b["x"] is None:
            raise RuntimeError("backward() needs a forward_train() first")
        sh, dev, st = self.shape, self.device, self.dev_status
        N, d, I, K, T = sh.n_routed, sh.d, sh.inter, sh.topk, sh.T
        R = T * K + T
        u8, f32, i32 = torch.uint8, torch.float32, torch.int32
        w2t, w2t_s, w13t, w13t_s = self._transposed_weights(stream)
        cuda_stream = (torch.cuda.current_stream(dev) if stream is None else
                       torch.cuda.ExternalStream(stream) if isinstance(stream, int) else stream)

        def mark(name):
            if marks is not None:
                ev = torch.cuda.Event(enable_timing=True)
                ev.record(cuda_stream)
                marks.append((name, ev))
        mark("start")
        off = self.expert_offsets
        do_q = torch.empty((R, d), dtype=u8, device=dev)
        do_s = torch.empty((d // 128, R), dtype=f32, device=dev)
        moe_combine_backward_quant(sh, dy, self.row_of_pair, self.topk_gate, do_q, do_s, st,
                                   stream)
        mark("combine_backward_quant")
        dh = torch.empty((R, I), dtype=f32, device=dev)
        moe_grouped_gemm_fp8(N + 1, off, R, do_q, do_s, d, w2t, w2t_s, I, MOE_EPI_F32, dh, None,
                             st, stream)
        mark("gemm_dh")
        ac = torch.empty((R, 2 * I), dtype=f32, device=dev)
        moe_grouped_gemm_fp8(N + 1, off, R, b["xq"], b["xs"], d, self.w13, self.w13_scales,
                             2 * I, MOE_EPI_F32, ac, None, st, stream)
        mark("gemm_ac_recompute")
        gq = torch.empty((R, 2 * I), dtype=u8, device=dev)
        gs = torch.empty((2 * I // 128, R), dtype=f32, device=dev)
        moe_swiglu_backward_quant(dh, ac, R, I, R, gq, gs, st, stream)
        mark("swiglu_backward_quant")
        dx_rows = torch.empty((R, d), dtype=f32, device=dev)
        moe_grouped_gemm_fp8(N + 1, off, R, gq, gs, 2 * I, w13t, w13t_s, d, MOE_EPI_F32,
                             dx_rows, None, st, stream)
        mark("gemm_dx")
        dgate = torch.empty((T, K), dtype=f32, device=dev)
        du = torch.empty((T, K), dtype=f32, device=dev)
        moe_gate_backward(sh, dy, b["o"], self.row_of_pair, b["score"], dgate, du, st, stream)
        mark("gate_backward")
        dx_router = torch.empty((T, d), dtype=f32, device=dev)
        d_router_w = torch.empty((N, d), dtype=f32, device=dev)
        pair_scratch = torch.empty((max(T * K, 1),), dtype=i32, device=dev)
        rbw = torch.empty((max(moe_router_backward_workspace_size(sh), 256),), dtype=u8,
                          device=dev)
        moe_router_backward(sh, b["x"], self.router_w, du, self.topk_idx, off, self.row_of_pair,
                            pair_scratch, dx_router, d_router_w, rbw, st, stream)
        mark("router_backward")
        dx = torch.empty((T, d), dtype=f32, device=dev)
        moe_dx_combine(sh, dx_rows, dx_router, self.row_of_pair, dx, st, stream)
        mark("dx_combine")
        self.last_dgate, self.last_du = dgate, du
        if not wgrad:
            return dx, d_router_w
        # ---- weight gradients (pair_scratch holds the permutation's inverse)
        G = N + 1
        nb = moe_wgrad_max_blocks(R, G)
        kb_off = torch.empty((G + 1,), dtype=i32, device=dev)
        blocks = torch.empty((nb, 2), dtype=i32, device=dev)
        moe_wgrad_layout(G, off, kb_off, blocks, st, stream)
        KP = nb * 128
        xt = torch.empty((d, KP), dtype=u8, device=dev)
        xts = torch.empty((nb, d), dtype=f32, device=dev)
        dact = torch.empty((2 * I, KP), dtype=u8, device=dev)
        dacts = torch.empty((nb, 2 * I), dtype=f32, device=dev)
        if T > 0:  # with no rows no group has K blocks: the operands are never read
            moe_wgrad_quant_x(sh, b["x"], pair_scratch, blocks, xt, xts, st, stream)
            moe_wgrad_quant_dac(dh, ac, I, blocks, dact, dacts, st, stream)
        mark("wgrad_quant_x_dac")
        dW13 = torch.empty((G, 2 * I, d), dtype=f32, device=dev)
        moe_grouped_gemm_wgrad(G, kb_off, nb, dact, dacts, 2 * I, xt, xts, d, dW13, st, stream)
        mark("gemm_dw13")
        del xt, xts, dact, dacts
        dot = torch.empty((d, KP), dtype=u8, device=dev)
        dots = torch.empty((nb, d), dtype=f32, device=dev)
        ht = torch.empty((I, KP), dtype=u8, device=dev)
        hts = torch.empty((nb, I), dtype=f32, device=dev)
        if T > 0:
            moe_wgrad_quant_do(sh, dy, self.topk_gate, pair_scratch, blocks, dot, dots, st,
                               stream)
            moe_wgrad_quant_h(ac, I, blocks, ht, hts, st, stream)
        mark("wgrad_quant_do_h")
        dW2 = torch.empty((G, d, I), dtype=f32, device=dev)
        moe_grouped_gemm_wgrad(G, kb_off, nb, dot, dots, d, ht, hts, I, dW2, st, stream)
        mark("gemm_dw2")
        return dx, d_router_w, dW13, dW2

    def status(self, stream=None) -> int:
        """Device status word (0 = fine); synchronises the stream."""
        return moe_read_status(self.dev_status, stream)
