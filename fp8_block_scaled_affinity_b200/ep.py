"""Expert-parallel MoE layer: one process per GPU, rank q owning routed
experts [q E, (q+1) E) with E = N_r / P, every rank running the shared expert
on its own tokens ("DeepSeek-V3 Technical Report" notes page, section
"DualPipe": all-to-all dispatch and combine around the expert MLP, tokens
sent to at most M nodes; section "FP8 mixed precision training": FP8
dispatch).

Every compute step runs in the library's kernels (routing, the dispatch plan,
quantise-and-pack into per-destination rows, the local permutation, the
grouped FP8 GEMMs, the partial and final combines); this module only drives
them and the exchanges: the counts and the rows of the dispatch and the fp32
partial outputs of the combine cross ranks with NCCL all-to-alls
(torch.distributed), whose split sizes need the per-destination counts on
the host (one small device-to-host copy per layer call).

`EpMoeLayer` holds one rank's state and exposes the stages; `ep_forward`
runs them with torch.distributed collectives.  The stages are separate so
that a caller may drive the exchange itself (for example several ranks'
stages in one process, each exchange a local copy)."""
from __future__ import annotations

from typing import Callable, Optional

from . import _lib
from ._lib import (MOE_EPI_F32, MOE_EPI_SWIGLU_QUANT, make_shape, moe_combine,  # noqa: F401
                   moe_ep_dispatch_plan, moe_ep_final_combine, moe_ep_local_permute,
                   moe_ep_pack, moe_ep_partial_combine, moe_ep_row_bytes,
                   moe_ep_workspace_size, moe_grouped_gemm_fp8, moe_route,
                   moe_route_workspace_size, moe_update_bias, fp8_quant_act_1x128,
                   fp8_quant_w_128x128)


def _mark(marks, name, device):
    """Append (name, CUDA event recorded on the current stream) when timing."""
    if marks is not None:
        import torch
        ev = torch.cuda.Event(enable_timing=True)
        ev.record(torch.cuda.current_stream(device))
        marks.append((name, ev))


class EpMoeLayer:
    """One rank's share of an expert-parallel MoE layer.

    shape: the layer's MoeShape with T = this rank's tokens per call (the
    ranks may differ in T).  Weights: routed experts of this rank plus the
    shared expert, FP8 with 128x128 FP32 scales (the pages' recipe)."""

    def __init__(self, shape, rank: int, n_ranks: int, router_w, bias, device=None):
        import torch
        if shape.n_routed % n_ranks:
            raise ValueError("n_routed must be a multiple of the number of ranks")
        self.shape, self.rank, self.P = shape, int(rank), int(n_ranks)
        self.E = shape.n_routed // n_ranks
        dev = torch.device(device) if device is not None else router_w.device
        self.device = dev
        d, I, N, K, T = shape.d, shape.inter, shape.n_routed, shape.topk, shape.T
        u8, f32, i32 = torch.uint8, torch.float32, torch.int32
        self.router_w, self.bias = router_w, bias
        # local experts 0..E-1, then the shared expert
        self.w13 = torch.empty((self.E + 1, 2 * I, d), dtype=u8, device=dev)
        self.w13_scales = torch.empty((self.E + 1, 2 * I // 128, d // 128), dtype=f32, device=dev)
        self.w2 = torch.empty((self.E + 1, d, I), dtype=u8, device=dev)
        self.w2_scales = torch.empty((self.E + 1, d // 128, I // 128), dtype=f32, device=dev)
        self.topk_idx = torch.empty((T, K), dtype=i32, device=dev)
        self.topk_gate = torch.empty((T, K), dtype=f32, device=dev)
        self.counts = torch.empty((N,), dtype=i32, device=dev)
        self.send_counts = torch.empty((self.P,), dtype=i32, device=dev)
        self.send_offsets = torch.empty((self.P + 1,), dtype=i32, device=dev)
        self.send_row = torch.empty((max(T, 1), self.P), dtype=i32, device=dev)
        self.route_ws = torch.empty((max(moe_route_workspace_size(shape), 256),), dtype=u8,
                                    device=dev)
        self.dev_status = torch.zeros((1,), dtype=i32, device=dev)
        self.row_bytes = moe_ep_row_bytes(shape)

    # ---------------------------------------------------------- weights
    def owns(self, e: int) -> bool:
        return e == self.shape.n_routed or self.rank * self.E <= e < (self.rank + 1) * self.E

    def set_expert(self, e: int, w1, w3, w2, stream=None) -> None:
        """Quantise expert e (global index; N_r = the shared expert) into this
        rank's buffers if this rank holds it."""
        if not self.owns(e):
            return
        j = self.E if e == self.shape.n_routed else e - self.rank * self.E
        I = self.shape.inter
        fp8_quant_w_128x128(w1, self.w13[j, :I], self.w13_scales[j, :I // 128], stream=stream)
        fp8_quant_w_128x128(w3, self.w13[j, I:], self.w13_scales[j, I // 128:], stream=stream)
        fp8_quant_w_128x128(w2, self.w2[j], self.w2_scales[j], stream=stream)

    # ---------------------------------------------------------- stages
    def route_and_pack(self, x, logit_offset=None, marks=None):
        """Routing with the (replicated) bias, the dispatch plan and the send
        rows.  Returns (send_buf, send_counts as a host list).  marks: as in
        MoeLayer.backward (events after "route", "plan", "pack")."""
        import torch
        sh, dev = self.shape, self.device
        _mark(marks, "start", dev)
        moe_route(sh, x, self.router_w, self.bias, logit_offset, self.topk_idx, self.topk_gate,
                  self.counts, self.route_ws, self.dev_status)
        _mark(marks, "route", dev)
        ws = torch.empty((moe_ep_workspace_size(sh, self.P, 0),), dtype=torch.uint8,
                         device=self.device)
        moe_ep_dispatch_plan(sh, self.P, self.topk_idx, self.send_counts, self.send_offsets,
                             self.send_row, ws, self.dev_status)
        _mark(marks, "plan", dev)
        counts = self.send_counts.cpu().tolist()  # split sizes for the exchange
        send_buf = torch.empty((max(sum(counts), 1), self.row_bytes), dtype=torch.uint8,
                               device=self.device)
        _mark(marks, "counts_to_host", dev)
        moe_ep_pack(sh, self.P, x, self.topk_idx, self.topk_gate, self.send_row, send_buf,
                    self.dev_status)
        _mark(marks, "pack", dev)
        return send_buf, counts

    def experts(self, recv_buf, n_recv: int, marks=None):
        """The local experts on the received rows; returns the fp32 partial
        outputs [n_recv, d] to send back (same row order).  marks: events
        after "local_permute", "gemm_w13", "gemm_w2", "partial_combine"."""
        import torch
        sh, dev = self.shape, self.device
        _mark(marks, "start", dev)
        d, I, K = sh.d, sh.inter, sh.topk
        max_rows = max(n_recv * min(K, self.E), 1)
        xq = torch.empty((max_rows, d), dtype=torch.uint8, device=dev)
        xs = torch.empty((d // 128, max_rows), dtype=torch.float32, device=dev)
        off = torch.empty((self.E + 1,), dtype=torch.int32, device=dev)
        pair_row = torch.empty((max(n_recv, 1), K), dtype=torch.int32, device=dev)
        ws = torch.empty((moe_ep_workspace_size(sh, self.P, n_recv),), dtype=torch.uint8,
                         device=dev)
        moe_ep_local_permute(sh, self.P, recv_buf, n_recv, xq, xs, max_rows, off, pair_row, ws,
                             self.dev_status)
        _mark(marks, "local_permute", dev)
        back = torch.empty((max(n_recv, 1), d), dtype=torch.float32, device=dev)
        if n_recv == 0:
            return back[:0]
        hq = torch.empty((max_rows, I), dtype=torch.uint8, device=dev)
        hs = torch.empty((I // 128, max_rows), dtype=torch.float32, device=dev)
        o = torch.empty((max_rows, d), dtype=torch.float32, device=dev)
        moe_grouped_gemm_fp8(self.E, off, max_rows, xq, xs, d, self.w13, self.w13_scales,
                             2 * I, MOE_EPI_SWIGLU_QUANT, hq, hs, self.dev_status)
        _mark(marks, "gemm_w13", dev)
        moe_grouped_gemm_fp8(self.E, off, max_rows, hq, hs, I, self.w2, self.w2_scales, d,
                             MOE_EPI_F32, o, None, self.dev_status)
        _mark(marks, "gemm_w2", dev)
        moe_ep_partial_combine(sh, self.P, recv_buf, n_recv, pair_row, o, back,
                               self.dev_status)
        _mark(marks, "partial_combine", dev)
        return back[:n_recv]

    def shared_and_combine(self, x, back_recv, marks=None):
        """The shared expert on this rank's tokens, then y = its output + the
        partial outputs of each token's destinations (rank order), bf16.
        marks: events after "shared_expert" and "final_combine"."""
        import torch
        sh, dev = self.shape, self.device
        _mark(marks, "start", dev)
        T, d, I = sh.T, sh.d, sh.inter
        y = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
        if T == 0:
            return y
        xq = torch.empty((T, d), dtype=torch.uint8, device=dev)
        xs = torch.empty((d // 128, T), dtype=torch.float32, device=dev)
        fp8_quant_act_1x128(x, xq, xs, True)
        off = torch.tensor([0, T], dtype=torch.int32, device=dev)
        hq = torch.empty((T, I), dtype=torch.uint8, device=dev)
        hs = torch.empty((I // 128, T), dtype=torch.float32, device=dev)
        o = torch.empty((T, d), dtype=torch.float32, device=dev)
        s = self.E  # the shared expert's slot
        moe_grouped_gemm_fp8(1, off, T, xq, xs, d, self.w13[s:], self.w13_scales[s:], 2 * I,
                             MOE_EPI_SWIGLU_QUANT, hq, hs, self.dev_status)
        moe_grouped_gemm_fp8(1, off, T, hq, hs, I, self.w2[s:], self.w2_scales[s:], d,
                             MOE_EPI_F32, o, None, self.dev_status)
        _mark(marks, "shared_expert", dev)
        moe_ep_final_combine(sh, self.P, o, back_recv if back_recv.numel() else None,
                             self.send_row, y, self.dev_status)
        _mark(marks, "final_combine", dev)
        return y

    def update_bias(self, global_counts, total_tokens: int) -> None:
        """b -/+ gamma from the load of the whole batch (all ranks' tokens)."""
        sh = self.shape
        g = make_shape(total_tokens, sh.d, sh.n_routed, sh.n_groups, sh.topk_groups, sh.topk,
                       sh.inter, sh.gamma)
        moe_update_bias(g, global_counts, self.bias, self.dev_status)


def ep_forward(layer: EpMoeLayer, x, group=None, logit_offset=None, update_bias=False,
               all_to_all: Optional[Callable] = None):
    """One expert-parallel layer call on this rank (all ranks call it together).

    The exchanges use torch.distributed (NCCL for CUDA tensors):
    all_to_all_single of the per-destination row counts, of the FP8 rows,
    and (reversed splits) of the fp32 partial outputs; with update_bias the
    expert counts are summed over the ranks first.  Returns y (bf16 [T, d])."""
    import torch
    import torch.distributed as dist
    a2a = all_to_all or (lambda out, inp, osz, isz: dist.all_to_all_single(
        out, inp, osz, isz, group=group))
    dev = layer.device
    send_buf, send_counts = layer.route_and_pack(x, logit_offset)
    sc = torch.tensor(send_counts, dtype=torch.int64, device=dev)
    rc = torch.empty_like(sc)
    a2a(rc, sc, None, None)
    recv_counts = rc.cpu().tolist()
    n_recv = sum(recv_counts)
    rb = layer.row_bytes
    recv_buf = torch.empty((max(n_recv, 1), rb), dtype=torch.uint8, device=dev)
    a2a(recv_buf[:n_recv].view(-1), send_buf[:sum(send_counts)].view(-1),
        [c * rb for c in recv_counts], [c * rb for c in send_counts])
    back = layer.experts(recv_buf, n_recv)
    back_recv = torch.empty((max(sum(send_counts), 1), layer.shape.d), dtype=back.dtype,
                            device=dev)
    d = layer.shape.d
    a2a(back_recv[:sum(send_counts)].view(-1), back.reshape(-1),
        [c * d for c in send_counts], [c * d for c in recv_counts])
    y = layer.shared_and_combine(x, back_recv[:sum(send_counts)])
    if update_bias:
        g = layer.counts.clone()
        dist.all_reduce(g, group=group)
        t = torch.tensor([layer.shape.T], dtype=torch.int64, device=dev)
        dist.all_reduce(t, group=group)
        layer.update_bias(g, int(t.item()))
    return y
