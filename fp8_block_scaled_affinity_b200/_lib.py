"""ctypes binding of libmoefp8.so (the C ABI declared in include/moefp8.h).

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels.  Functions keep the C names; tensors are torch tensors on the
current CUDA device (their data pointers are passed), and `stream` defaults to
torch's current stream.  A non-zero status raises MoeError.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoefp8.so")

MOE_OK = 0
MOE_EPI_F32 = 0
MOE_EPI_BF16 = 1
MOE_EPI_SWIGLU_QUANT = 2
MOE_DEV_TIMEOUT = 1


class MoeError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: status {status} ({status_string(status)})")


class MoeShape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int), ("d", ctypes.c_int), ("n_routed", ctypes.c_int),
                ("n_groups", ctypes.c_int), ("topk_groups", ctypes.c_int),
                ("topk", ctypes.c_int), ("inter", ctypes.c_int), ("gamma", ctypes.c_float)]


class MoeWeights(ctypes.Structure):
    _fields_ = [("w13", ctypes.c_void_p), ("w13_scales", ctypes.c_void_p),
                ("w2", ctypes.c_void_p), ("w2_scales", ctypes.c_void_p),
                ("router_w", ctypes.c_void_p)]


class MoeWeightsMx(ctypes.Structure):
    _fields_ = [("w13", ctypes.c_void_p), ("w13_sf", ctypes.c_void_p),
                ("w2", ctypes.c_void_p), ("w2_sf", ctypes.c_void_p),
                ("router_w", ctypes.c_void_p)]


class MoeRouting(ctypes.Structure):
    _fields_ = [("topk_idx", ctypes.c_void_p), ("topk_gate", ctypes.c_void_p),
                ("expert_counts", ctypes.c_void_p), ("expert_offsets", ctypes.c_void_p),
                ("row_of_pair", ctypes.c_void_p)]


_L = None


def lib() -> ctypes.CDLL:
    """Load libmoefp8.so (built in-tree by __graft_entry__.build()).  Raises
    if it is missing: there is no fallback implementation."""
    global _L
    if _L is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with "
                              "`python -c 'import __graft_entry__ as g; g.build()'`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        SP = ctypes.POINTER(MoeShape)
        sig = {
            "moe_version": (I, []),
            "moe_status_string": (ctypes.c_char_p, [I]),
            "moe_read_status": (I, [P, P, P]),
            "moe_route_workspace_size": (SZ, [SP]),
            "moe_route": (I, [SP, P, P, P, P, P, P, P, P, SZ, P, P]),
            "moe_route_scores": (I, [SP, P, P, P, P, P, P, P, P, P, SZ, P, P]),
            "fp8_transpose_w_128x128": (I, [P, P, I64, I64, I64, P, P, P, P]),
            "moe_combine_backward_quant": (I, [SP, P, P, P, P, P, P, P]),
            "moe_swiglu_backward_quant": (I, [P, P, I64, I, I64, P, P, P, P]),
            "moe_gate_backward": (I, [SP, P, P, P, P, P, P, P, P]),
            "moe_router_backward_workspace_size": (SZ, [SP]),
            "moe_router_backward": (I, [SP, P, P, P, P, P, P, P, P, P, P, SZ, P, P]),
            "moe_dx_combine": (I, [SP, P, P, P, P, P, P]),
            "moe_wgrad_max_blocks": (I, [I64, I]),
            "moe_wgrad_layout": (I, [I, P, I, P, P, P, P]),
            "moe_wgrad_quant_x": (I, [SP, P, P, P, I, P, P, P, P]),
            "moe_wgrad_quant_do": (I, [SP, P, P, P, P, I, P, P, P, P]),
            "moe_wgrad_quant_h": (I, [P, I, P, I, P, P, P, P]),
            "moe_wgrad_quant_dac": (I, [P, P, I, P, I, P, P, P, P]),
            "moe_grouped_gemm_wgrad": (I, [I, P, I, P, P, I, P, P, I, P, P, P]),
            "fp8_quant_act_1x128": (I, [P, I64, I64, P, P, I, P, P]),
            "fp8_quant_w_128x128": (I, [P, I64, I64, P, P, P, P]),
            "moe_permute_workspace_size": (SZ, [SP]),
            "moe_permute": (I, [SP, P, P, P, P, P, P, P, P, P, SZ, P, P]),
            "moe_permute_static_ws": (I, [SP, P, P, P, P, P, P, P, P, P, P]),
            "moe_quant_permute": (I, [SP, P, P, P, P, P, P, P, P, SZ, P, P]),
            "moe_grouped_gemm_fp8": (I, [I, P, I, P, P, I, P, P, I, I, P, P, P, P]),
            "moe_grouped_gemm_form": (I, [I, I, I, I]),
            "fp8_quant_act_1x128_ue8m0": (I, [P, I64, I64, P, P, I, P, P]),
            "fp8_quant_w_128x128_ue8m0": (I, [P, I64, I64, P, P, P, P]),
            "moe_grouped_gemm_mxfp8": (I, [I, P, I, P, P, I, P, P, I, I, P, P, P, P]),
            "moe_grouped_gemm_fp8_indexed": (I, [I, P, P, I, I, P, P, I, P, P, I, I, P, P, P,
                                                 P]),
            "moe_plan_redundant_experts": (I, [P, I, I, P, P]),
            "moe_quant_permute_ue8m0": (I, [SP, P, P, P, P, P, P, P, P, SZ, P, P]),
            "moe_ep_row_bytes": (SZ, [SP]),
            "moe_ep_workspace_size": (SZ, [SP, I, I]),
            "moe_ep_dispatch_plan": (I, [SP, I, P, P, P, P, P, SZ, P, P]),
            "moe_ep_pack": (I, [SP, I, P, P, P, P, P, P, P]),
            "moe_ep_local_permute": (I, [SP, I, P, I, P, P, I, P, P, P, SZ, P, P]),
            "moe_ep_partial_combine": (I, [SP, I, P, I, P, P, P, P, P]),
            "moe_ep_final_combine": (I, [SP, I, P, P, P, P, P, P]),
            "moe_layer_mx_workspace_size": (SZ, [SP]),
            "moe_layer_forward_mx": (I, [SP, ctypes.POINTER(MoeWeightsMx), P, P, P,
                                         ctypes.POINTER(MoeRouting), P, I, P, SZ, P, P]),
            "moe_split_groups": (I, [SP, P, P, P, P, I, P, P, P, P]),
            "moe_combine": (I, [SP, P, P, P, P, P, P, P]),
            "moe_update_bias": (I, [SP, P, P, P, P]),
            "moe_layer_workspace_size": (SZ, [SP]),
            "moe_layer_forward": (I, [SP, ctypes.POINTER(MoeWeights), P, P, P,
                                      ctypes.POINTER(MoeRouting), P, I, P, SZ, P, P]),
            "moe_layer_host_workspace_size": (SZ, [SP]),
            "moe_layer_forward_host": (I, [SP, ctypes.POINTER(MoeWeights), P, P, P,
                                           ctypes.POINTER(MoeRouting), P, I, P, SZ, P, P]),
            "moe_layer_host_batches_workspace_size": (SZ, [SP]),
            "moe_layer_forward_host_batches": (I, [SP, ctypes.POINTER(MoeWeights), P, I, P, P,
                                                   ctypes.POINTER(MoeRouting), P, I, P, SZ, P,
                                                   P]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _L = L
    return _L


def status_string(status: int) -> str:
    return lib().moe_status_string(int(status)).decode()


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(name: str, rc: int) -> None:
    if rc != MOE_OK:
        raise MoeError(name, rc)


def make_shape(T, d, n_routed, n_groups, topk_groups, topk, inter, gamma=0.001) -> MoeShape:
    return MoeShape(int(T), int(d), int(n_routed), int(n_groups), int(topk_groups), int(topk),
                    int(inter), float(gamma))


def moe_version() -> int:
    return lib().moe_version()


def moe_read_status(dev_status, stream=None) -> int:
    out = ctypes.c_int(0)
    _check("moe_read_status", lib().moe_read_status(_ptr(dev_status), ctypes.addressof(out),
                                                    _stream(stream)))
    return out.value


def moe_route_workspace_size(shape: MoeShape) -> int:
    return lib().moe_route_workspace_size(ctypes.byref(shape))


def moe_route(shape, x, router_w, bias, logit_offset, topk_idx, topk_gate, expert_counts,
              ws, dev_status=None, stream=None) -> None:
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check("moe_route", lib().moe_route(
        ctypes.byref(shape), _ptr(x), _ptr(router_w), _ptr(bias), _ptr(logit_offset),
        _ptr(topk_idx), _ptr(topk_gate), _ptr(expert_counts), _ptr(ws), nbytes,
        _ptr(dev_status), _stream(stream)))


def moe_route_scores(shape, x, router_w, bias, logit_offset, topk_idx, topk_gate, topk_score,
                     expert_counts, ws, dev_status=None, stream=None) -> None:
    """moe_route that also returns the chosen unbiased affinities (topk_score)."""
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check("moe_route_scores", lib().moe_route_scores(
        ctypes.byref(shape), _ptr(x), _ptr(router_w), _ptr(bias), _ptr(logit_offset),
        _ptr(topk_idx), _ptr(topk_gate), _ptr(topk_score), _ptr(expert_counts), _ptr(ws),
        nbytes, _ptr(dev_status), _stream(stream)))


def fp8_quant_act_1x128(x, q, scales, scales_kb_major=False, dev_status=None, stream=None):
    rows, cols = x.shape
    _check("fp8_quant_act_1x128", lib().fp8_quant_act_1x128(
        _ptr(x), rows, cols, _ptr(q), _ptr(scales), int(bool(scales_kb_major)),
        _ptr(dev_status), _stream(stream)))


def fp8_quant_w_128x128(w, q, scales, dev_status=None, stream=None):
    rows, cols = w.shape
    _check("fp8_quant_w_128x128", lib().fp8_quant_w_128x128(
        _ptr(w), rows, cols, _ptr(q), _ptr(scales), _ptr(dev_status), _stream(stream)))


def moe_permute_workspace_size(shape: MoeShape) -> int:
    return lib().moe_permute_workspace_size(ctypes.byref(shape))


def moe_permute(shape, topk_idx, expert_counts, xq, xs, xq_perm, xs_perm, expert_offsets,
                row_of_pair, ws, dev_status=None, stream=None):
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check("moe_permute", lib().moe_permute(
        ctypes.byref(shape), _ptr(topk_idx), _ptr(expert_counts), _ptr(xq), _ptr(xs),
        _ptr(xq_perm), _ptr(xs_perm), _ptr(expert_offsets), _ptr(row_of_pair), _ptr(ws), nbytes,
        _ptr(dev_status), _stream(stream)))


def moe_quant_permute(shape, x, topk_idx, expert_counts, xq_perm, xs_perm, expert_offsets,
                      row_of_pair, ws, dev_status=None, stream=None):
    """fp8_quant_act_1x128 of x (bf16 [T, d]) fused with moe_permute."""
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check("moe_quant_permute", lib().moe_quant_permute(
        ctypes.byref(shape), _ptr(x), _ptr(topk_idx), _ptr(expert_counts), _ptr(xq_perm),
        _ptr(xs_perm), _ptr(expert_offsets), _ptr(row_of_pair), _ptr(ws), nbytes,
        _ptr(dev_status), _stream(stream)))


def moe_permute_static_ws(shape, topk_idx, expert_counts, xq, xs, xq_perm, xs_perm,
                          expert_offsets, row_of_pair, dev_status=None, stream=None):
    """moe_permute for callers that cannot allocate device memory while they
    run: no workspace argument; the library's own fixed 1 MiB device array
    is used instead (ceil(T/64) * N_r <= 262144).  Calls that overlap on the
    GPU share that array and race."""
    _check("moe_permute_static_ws", lib().moe_permute_static_ws(
        ctypes.byref(shape), _ptr(topk_idx), _ptr(expert_counts), _ptr(xq), _ptr(xs),
        _ptr(xq_perm), _ptr(xs_perm), _ptr(expert_offsets), _ptr(row_of_pair),
        _ptr(dev_status), _stream(stream)))


def moe_grouped_gemm_fp8(n_groups, group_offsets, max_rows, a, a_scales, k, w, w_scales, n,
                         epilogue, out, out_scales=None, dev_status=None, stream=None):
    _check("moe_grouped_gemm_fp8", lib().moe_grouped_gemm_fp8(
        int(n_groups), _ptr(group_offsets), int(max_rows), _ptr(a), _ptr(a_scales), int(k),
        _ptr(w), _ptr(w_scales), int(n), int(epilogue), _ptr(out), _ptr(out_scales),
        _ptr(dev_status), _stream(stream)))


def moe_grouped_gemm_form(n_groups, max_rows, n, epilogue) -> int:
    """CTAs per tile moe_grouped_gemm_fp8 uses for these arguments on the
    current device: 1 (single CTAs), 2 (CTA pairs), 0 (invalid arguments)."""
    return int(lib().moe_grouped_gemm_form(int(n_groups), int(max_rows), int(n), int(epilogue)))


def moe_combine(shape, expert_out, expert_offsets, row_of_pair, topk_gate, y,
                dev_status=None, stream=None):
    _check("moe_combine", lib().moe_combine(
        ctypes.byref(shape), _ptr(expert_out), _ptr(expert_offsets), _ptr(row_of_pair),
        _ptr(topk_gate), _ptr(y), _ptr(dev_status), _stream(stream)))


def moe_update_bias(shape, expert_counts, bias, dev_status=None, stream=None):
    _check("moe_update_bias", lib().moe_update_bias(
        ctypes.byref(shape), _ptr(expert_counts), _ptr(bias), _ptr(dev_status),
        _stream(stream)))


def moe_layer_workspace_size(shape: MoeShape) -> int:
    return lib().moe_layer_workspace_size(ctypes.byref(shape))


def moe_layer_host_workspace_size(shape: MoeShape) -> int:
    return lib().moe_layer_host_workspace_size(ctypes.byref(shape))


def make_weights(w13, w13_scales, w2, w2_scales, router_w) -> MoeWeights:
    return MoeWeights(_ptr(w13), _ptr(w13_scales), _ptr(w2), _ptr(w2_scales), _ptr(router_w))


def make_routing(topk_idx, topk_gate, expert_counts, expert_offsets, row_of_pair) -> MoeRouting:
    return MoeRouting(_ptr(topk_idx), _ptr(topk_gate), _ptr(expert_counts),
                      _ptr(expert_offsets), _ptr(row_of_pair))


def moe_layer_forward(shape, weights: MoeWeights, x, bias, logit_offset, routing: MoeRouting,
                      y, update_bias, ws, dev_status=None, stream=None):
    nbytes = ws.numel() * ws.element_size()
    _check("moe_layer_forward", lib().moe_layer_forward(
        ctypes.byref(shape), ctypes.byref(weights), _ptr(x), _ptr(bias), _ptr(logit_offset),
        ctypes.byref(routing), _ptr(y), int(bool(update_bias)), _ptr(ws), nbytes,
        _ptr(dev_status), _stream(stream)))


def moe_layer_forward_host(shape, weights: MoeWeights, x_host, bias, logit_offset,
                           routing: MoeRouting, y_host, update_bias, ws, dev_status=None,
                           stream=None):
    nbytes = ws.numel() * ws.element_size()
    _check("moe_layer_forward_host", lib().moe_layer_forward_host(
        ctypes.byref(shape), ctypes.byref(weights), _ptr(x_host), _ptr(bias),
        _ptr(logit_offset), ctypes.byref(routing), _ptr(y_host), int(bool(update_bias)),
        _ptr(ws), nbytes, _ptr(dev_status), _stream(stream)))


def moe_layer_host_batches_workspace_size(shape: MoeShape) -> int:
    return lib().moe_layer_host_batches_workspace_size(ctypes.byref(shape))


def moe_layer_forward_host_batches(shape, weights: MoeWeights, x_host, n_batches, bias,
                                   logit_offset, routing: MoeRouting, y_host, update_bias, ws,
                                   dev_status=None, stream=None):
    """n_batches successive batches, x_host / y_host pinned [n_batches, T, d]."""
    nbytes = ws.numel() * ws.element_size()
    _check("moe_layer_forward_host_batches", lib().moe_layer_forward_host_batches(
        ctypes.byref(shape), ctypes.byref(weights), _ptr(x_host), int(n_batches), _ptr(bias),
        _ptr(logit_offset), ctypes.byref(routing), _ptr(y_host), int(bool(update_bias)),
        _ptr(ws), nbytes, _ptr(dev_status), _stream(stream)))


# ------------------------------------------- power-of-two scale option
def fp8_quant_act_1x128_ue8m0(x, q, sf, sf_kb_major=False, dev_status=None, stream=None):
    """1x128 tiles with power-of-two scales; sf: uint8 UE8M0 bytes."""
    rows, cols = x.shape
    _check("fp8_quant_act_1x128_ue8m0", lib().fp8_quant_act_1x128_ue8m0(
        _ptr(x), rows, cols, _ptr(q), _ptr(sf), int(bool(sf_kb_major)), _ptr(dev_status),
        _stream(stream)))


def fp8_quant_w_128x128_ue8m0(w, q, sf, dev_status=None, stream=None):
    rows, cols = w.shape
    _check("fp8_quant_w_128x128_ue8m0", lib().fp8_quant_w_128x128_ue8m0(
        _ptr(w), rows, cols, _ptr(q), _ptr(sf), _ptr(dev_status), _stream(stream)))


def moe_grouped_gemm_mxfp8(n_groups, group_offsets, max_rows, a, a_sf, k, w, w_sf, n, epilogue,
                           out, out_sf=None, dev_status=None, stream=None):
    _check("moe_grouped_gemm_mxfp8", lib().moe_grouped_gemm_mxfp8(
        int(n_groups), _ptr(group_offsets), int(max_rows), _ptr(a), _ptr(a_sf), int(k), _ptr(w),
        _ptr(w_sf), int(n), int(epilogue), _ptr(out), _ptr(out_sf), _ptr(dev_status),
        _stream(stream)))


# ----------------------------------------------------- redundant experts
def moe_grouped_gemm_fp8_indexed(n_groups, group_offsets, group_weight, n_weights, max_rows, a,
                                 a_scales, k, w, w_scales, n, epilogue, out, out_scales=None,
                                 dev_status=None, stream=None):
    _check("moe_grouped_gemm_fp8_indexed", lib().moe_grouped_gemm_fp8_indexed(
        int(n_groups), _ptr(group_offsets), _ptr(group_weight), int(n_weights), int(max_rows),
        _ptr(a), _ptr(a_scales), int(k), _ptr(w), _ptr(w_scales), int(n), int(epilogue),
        _ptr(out), _ptr(out_scales), _ptr(dev_status), _stream(stream)))


def moe_plan_redundant_experts(counts, n_extra):
    """Host planner: counts (sequence of ints) -> (replicas, slot_expert) as
    numpy int32 arrays."""
    import numpy as np
    c = np.ascontiguousarray(np.asarray(counts, dtype=np.int32))
    rep = np.empty(c.size, dtype=np.int32)
    slots = np.empty(c.size + int(n_extra), dtype=np.int32)
    _check("moe_plan_redundant_experts", lib().moe_plan_redundant_experts(
        c.ctypes.data, int(c.size), int(n_extra), rep.ctypes.data, slots.ctypes.data))
    return rep, slots


def moe_split_groups(shape, expert_offsets, replicas, slot_expert, first_slot, n_extra,
                     slot_offsets, slot_weight, dev_status=None, stream=None):
    _check("moe_split_groups", lib().moe_split_groups(
        ctypes.byref(shape), _ptr(expert_offsets), _ptr(replicas), _ptr(slot_expert),
        _ptr(first_slot), int(n_extra), _ptr(slot_offsets), _ptr(slot_weight), _ptr(dev_status),
        _stream(stream)))


def moe_quant_permute_ue8m0(shape, x, topk_idx, expert_counts, xq_perm, xsf_perm,
                            expert_offsets, row_of_pair, ws, dev_status=None, stream=None):
    """moe_quant_permute with power-of-two scales (xsf_perm: uint8 UE8M0)."""
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check("moe_quant_permute_ue8m0", lib().moe_quant_permute_ue8m0(
        ctypes.byref(shape), _ptr(x), _ptr(topk_idx), _ptr(expert_counts), _ptr(xq_perm),
        _ptr(xsf_perm), _ptr(expert_offsets), _ptr(row_of_pair), _ptr(ws), nbytes,
        _ptr(dev_status), _stream(stream)))


def moe_layer_mx_workspace_size(shape: MoeShape) -> int:
    return lib().moe_layer_mx_workspace_size(ctypes.byref(shape))


def make_weights_mx(w13, w13_sf, w2, w2_sf, router_w) -> MoeWeightsMx:
    return MoeWeightsMx(_ptr(w13), _ptr(w13_sf), _ptr(w2), _ptr(w2_sf), _ptr(router_w))


def moe_layer_forward_mx(shape, weights: MoeWeightsMx, x, bias, logit_offset,
                         routing: MoeRouting, y, update_bias, ws, dev_status=None, stream=None):
    nbytes = ws.numel() * ws.element_size()
    _check("moe_layer_forward_mx", lib().moe_layer_forward_mx(
        ctypes.byref(shape), ctypes.byref(weights), _ptr(x), _ptr(bias), _ptr(logit_offset),
        ctypes.byref(routing), _ptr(y), int(bool(update_bias)), _ptr(ws), nbytes,
        _ptr(dev_status), _stream(stream)))


# -------------------------------------------------- expert parallelism
def moe_ep_row_bytes(shape) -> int:
    return int(lib().moe_ep_row_bytes(ctypes.byref(shape)))


def moe_ep_workspace_size(shape, n_ranks, max_recv_rows) -> int:
    return int(lib().moe_ep_workspace_size(ctypes.byref(shape), int(n_ranks),
                                           int(max_recv_rows)))


def moe_ep_dispatch_plan(shape, n_ranks, topk_idx, send_counts, send_offsets, send_row, ws,
                         dev_status=None, stream=None):
    nbytes = ws.numel() * ws.element_size()
    _check("moe_ep_dispatch_plan", lib().moe_ep_dispatch_plan(
        ctypes.byref(shape), int(n_ranks), _ptr(topk_idx), _ptr(send_counts),
        _ptr(send_offsets), _ptr(send_row), _ptr(ws), nbytes, _ptr(dev_status),
        _stream(stream)))


def moe_ep_pack(shape, n_ranks, x, topk_idx, topk_gate, send_row, send_buf, dev_status=None,
                stream=None):
    _check("moe_ep_pack", lib().moe_ep_pack(
        ctypes.byref(shape), int(n_ranks), _ptr(x), _ptr(topk_idx), _ptr(topk_gate),
        _ptr(send_row), _ptr(send_buf), _ptr(dev_status), _stream(stream)))


def moe_ep_local_permute(shape, n_ranks, recv_buf, n_recv, xq_perm, xs_perm, max_rows,
                         local_offsets, pair_row, ws, dev_status=None, stream=None):
    nbytes = ws.numel() * ws.element_size()
    _check("moe_ep_local_permute", lib().moe_ep_local_permute(
        ctypes.byref(shape), int(n_ranks), _ptr(recv_buf), int(n_recv), _ptr(xq_perm),
        _ptr(xs_perm), int(max_rows), _ptr(local_offsets), _ptr(pair_row), _ptr(ws), nbytes,
        _ptr(dev_status), _stream(stream)))


def moe_ep_partial_combine(shape, n_ranks, recv_buf, n_recv, pair_row, expert_out, back_buf,
                           dev_status=None, stream=None):
    _check("moe_ep_partial_combine", lib().moe_ep_partial_combine(
        ctypes.byref(shape), int(n_ranks), _ptr(recv_buf), int(n_recv), _ptr(pair_row),
        _ptr(expert_out), _ptr(back_buf), _ptr(dev_status), _stream(stream)))


def moe_ep_final_combine(shape, n_ranks, shared_out, back_recv, send_row, y, dev_status=None,
                         stream=None):
    _check("moe_ep_final_combine", lib().moe_ep_final_combine(
        ctypes.byref(shape), int(n_ranks), _ptr(shared_out), _ptr(back_recv), _ptr(send_row),
        _ptr(y), _ptr(dev_status), _stream(stream)))


# ------------------------------------------------------------- backward
def fp8_transpose_w_128x128(q, scales, qt, scales_t, dev_status=None, stream=None):
    """q uint8 [mats, rows, cols] (or [rows, cols]), scales fp32
    [mats, rows/128, cols/128] -> the transposed codes and scales."""
    rows, cols = q.shape[-2], q.shape[-1]
    mats = q.numel() // max(rows * cols, 1) if rows * cols else 0
    _check("fp8_transpose_w_128x128", lib().fp8_transpose_w_128x128(
        _ptr(q), _ptr(scales), int(mats), int(rows), int(cols), _ptr(qt), _ptr(scales_t),
        _ptr(dev_status), _stream(stream)))


def moe_combine_backward_quant(shape, dy, row_of_pair, topk_gate, do_q, do_scales,
                               dev_status=None, stream=None):
    _check("moe_combine_backward_quant", lib().moe_combine_backward_quant(
        ctypes.byref(shape), _ptr(dy), _ptr(row_of_pair), _ptr(topk_gate), _ptr(do_q),
        _ptr(do_scales), _ptr(dev_status), _stream(stream)))


def moe_swiglu_backward_quant(dh, ac, rows, inter, rows_total, q, q_scales, dev_status=None,
                              stream=None):
    _check("moe_swiglu_backward_quant", lib().moe_swiglu_backward_quant(
        _ptr(dh), _ptr(ac), int(rows), int(inter), int(rows_total), _ptr(q), _ptr(q_scales),
        _ptr(dev_status), _stream(stream)))


def moe_gate_backward(shape, dy, expert_out, row_of_pair, topk_score, dgate, du,
                      dev_status=None, stream=None):
    _check("moe_gate_backward", lib().moe_gate_backward(
        ctypes.byref(shape), _ptr(dy), _ptr(expert_out), _ptr(row_of_pair), _ptr(topk_score),
        _ptr(dgate), _ptr(du), _ptr(dev_status), _stream(stream)))


def moe_router_backward_workspace_size(shape) -> int:
    return int(lib().moe_router_backward_workspace_size(ctypes.byref(shape)))


def moe_router_backward(shape, x, router_w, du, topk_idx, expert_offsets, row_of_pair,
                        pair_scratch, dx_router, d_router_w, ws, dev_status=None, stream=None):
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check("moe_router_backward", lib().moe_router_backward(
        ctypes.byref(shape), _ptr(x), _ptr(router_w), _ptr(du), _ptr(topk_idx),
        _ptr(expert_offsets), _ptr(row_of_pair), _ptr(pair_scratch), _ptr(dx_router),
        _ptr(d_router_w), _ptr(ws), nbytes, _ptr(dev_status), _stream(stream)))


def moe_dx_combine(shape, dx_rows, dx_router, row_of_pair, dx, dev_status=None, stream=None):
    _check("moe_dx_combine", lib().moe_dx_combine(
        ctypes.byref(shape), _ptr(dx_rows), _ptr(dx_router), _ptr(row_of_pair), _ptr(dx),
        _ptr(dev_status), _stream(stream)))


# ------------------------------------------------------- weight gradients
def moe_wgrad_max_blocks(rows, n_groups) -> int:
    return int(lib().moe_wgrad_max_blocks(int(rows), int(n_groups)))


def moe_wgrad_layout(n_groups, row_offsets, kb_offsets, blocks, dev_status=None, stream=None):
    """blocks: int32 [max_blocks, 2]."""
    _check("moe_wgrad_layout", lib().moe_wgrad_layout(
        int(n_groups), _ptr(row_offsets), int(blocks.shape[0]), _ptr(kb_offsets), _ptr(blocks),
        _ptr(dev_status), _stream(stream)))


def moe_wgrad_quant_x(shape, x, pair_of_row, blocks, xt, xt_scales, dev_status=None,
                      stream=None):
    _check("moe_wgrad_quant_x", lib().moe_wgrad_quant_x(
        ctypes.byref(shape), _ptr(x), _ptr(pair_of_row), _ptr(blocks), int(blocks.shape[0]),
        _ptr(xt), _ptr(xt_scales), _ptr(dev_status), _stream(stream)))


def moe_wgrad_quant_do(shape, dy, topk_gate, pair_of_row, blocks, dot, dot_scales,
                       dev_status=None, stream=None):
    _check("moe_wgrad_quant_do", lib().moe_wgrad_quant_do(
        ctypes.byref(shape), _ptr(dy), _ptr(topk_gate), _ptr(pair_of_row), _ptr(blocks),
        int(blocks.shape[0]), _ptr(dot), _ptr(dot_scales), _ptr(dev_status), _stream(stream)))


def moe_wgrad_quant_h(ac, inter, blocks, ht, ht_scales, dev_status=None, stream=None):
    _check("moe_wgrad_quant_h", lib().moe_wgrad_quant_h(
        _ptr(ac), int(inter), _ptr(blocks), int(blocks.shape[0]), _ptr(ht), _ptr(ht_scales),
        _ptr(dev_status), _stream(stream)))


def moe_wgrad_quant_dac(dh, ac, inter, blocks, dact, dact_scales, dev_status=None, stream=None):
    _check("moe_wgrad_quant_dac", lib().moe_wgrad_quant_dac(
        _ptr(dh), _ptr(ac), int(inter), _ptr(blocks), int(blocks.shape[0]), _ptr(dact),
        _ptr(dact_scales), _ptr(dev_status), _stream(stream)))


def moe_grouped_gemm_wgrad(n_groups, kb_offsets, nkb_total, a_t, a_scales, m, b_t, b_scales, n,
                           out, dev_status=None, stream=None):
    _check("moe_grouped_gemm_wgrad", lib().moe_grouped_gemm_wgrad(
        int(n_groups), _ptr(kb_offsets), int(nkb_total), _ptr(a_t), _ptr(a_scales), int(m),
        _ptr(b_t), _ptr(b_scales), int(n), _ptr(out), _ptr(dev_status), _stream(stream)))
