"""Python face of the CPU oracle: ctypes calls into moe_oracle.c for the
bit-exact steps (E4M3 codes, scales, routing, bias update, permutation
layout) and numpy FP64 for the expert matmuls and the combine.

TEST INFRASTRUCTURE ONLY (see the package docstring).
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Callable, Optional

import numpy as np

from . import build as _build

__all__ = [
    "lib", "e4m3_decode_table", "e4m3_encode", "quant_act_1x128",
    "quant_w_128x128", "dequant_act", "dequant_w", "route", "update_bias",
    "permute_layout", "swiglu_expert", "f64_to_bf16_bits", "combine",
    "quantized_expert", "layer_forward", "gemm_blockscaled",
    "quant_act_1x128_pow2", "quant_w_128x128_pow2", "pow2_scales",
    "redundant_plan", "split_groups", "quantized_expert_pow2", "quant_act_1x128_pow2_values",
    "gate_backward", "router_backward", "expert_backward", "layer_backward", "swiglu_backward",
    "quant_act_128x1", "gemm_wgrad",
]

_LIB = None


def lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I = ctypes.c_int
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_e4m3_encode.argtypes = [ctypes.c_float]
        L.orc_e4m3_encode_array.argtypes = [P, I64, P]
        L.orc_quant_act_1x128_bf16.argtypes = [P, I64, I64, P, P]
        L.orc_quant_act_1x128_f32.argtypes = [P, I64, I64, P, P]
        L.orc_quant_w_128x128.argtypes = [P, I64, I64, P, P]
        L.orc_quant_act_1x128_pow2_bf16.argtypes = [P, I64, I64, P, P]
        L.orc_quant_act_1x128_pow2_f32.argtypes = [P, I64, I64, P, P]
        L.orc_quant_w_128x128_pow2.argtypes = [P, I64, I64, P, P]
        L.orc_route.restype = I
        L.orc_route.argtypes = [I, I, I, I, I, I, P, P, P, P, P, P, P, P, P]
        L.orc_update_bias.argtypes = [I, I, I, P, ctypes.c_float, P]
        L.orc_permute_layout.argtypes = [I, I, I, P, P, P, P]
        _LIB = L
    return _LIB


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ------------------------------------------------------------------- E4M3
def e4m3_decode_table() -> np.ndarray:
    """FP64 value of each of the 256 E4M3 codes (NaN for the two NaN codes)."""
    L = lib()
    return np.array([L.orc_e4m3_decode(c) for c in range(256)], dtype=np.float64)


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    v = _c(v, np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().orc_e4m3_encode_array(_p(v), v.size, _p(out))
    return out


# ------------------------------------------------------------ quantisation
def quant_act_1x128(x: np.ndarray):
    """1x128 tile quantisation of a [rows, cols] matrix.

    ``x`` is either uint16 bf16 bits or float32.  Returns (codes uint8
    [rows, cols], scales float32 [rows, cols/128])."""
    rows, cols = x.shape
    assert cols % 128 == 0
    q = np.empty((rows, cols), dtype=np.uint8)
    s = np.empty((rows, cols // 128), dtype=np.float32)
    if x.dtype == np.uint16:
        x = _c(x, np.uint16)
        lib().orc_quant_act_1x128_bf16(_p(x), rows, cols, _p(q), _p(s))
    else:
        x = _c(x, np.float32)
        lib().orc_quant_act_1x128_f32(_p(x), rows, cols, _p(q), _p(s))
    return q, s


def quant_w_128x128(w: np.ndarray):
    """128x128 block quantisation of bf16 bits [rows, cols]."""
    rows, cols = w.shape
    assert rows % 128 == 0 and cols % 128 == 0
    w = _c(w, np.uint16)
    q = np.empty((rows, cols), dtype=np.uint8)
    s = np.empty((rows // 128, cols // 128), dtype=np.float32)
    lib().orc_quant_w_128x128(_p(w), rows, cols, _p(q), _p(s))
    return q, s


# ------------------------------------------- power-of-two scales (option)
# Not the pages' recipe (their scales are arbitrary FP32 values): a
# numerically different option whose scales are powers of two, so that
# block-scaled tensor-core MMAs with UE8M0 scale factors can apply them.
# Each function returns (codes, e) with e the int32 exponent of every scale
# (scale = 2^e, UE8M0 byte = e + 127).

def quant_act_1x128_pow2(x: np.ndarray):
    """1x128 tiles, scale 2^e with e the smallest integer such that
    amax <= 448 * 2^e; codes E4M3(v * 2^-e).  x: uint16 bf16 bits or fp32."""
    rows, cols = x.shape
    assert cols % 128 == 0
    q = np.empty((rows, cols), dtype=np.uint8)
    e = np.empty((rows, cols // 128), dtype=np.int32)
    if x.dtype == np.uint16:
        x = _c(x, np.uint16)
        lib().orc_quant_act_1x128_pow2_bf16(_p(x), rows, cols, _p(q), _p(e))
    else:
        x = _c(x, np.float32)
        lib().orc_quant_act_1x128_pow2_f32(_p(x), rows, cols, _p(q), _p(e))
    return q, e


def quant_w_128x128_pow2(w: np.ndarray):
    """128x128 blocks of bf16 bits [rows, cols] with power-of-two scales."""
    rows, cols = w.shape
    assert rows % 128 == 0 and cols % 128 == 0
    w = _c(w, np.uint16)
    q = np.empty((rows, cols), dtype=np.uint8)
    e = np.empty((rows // 128, cols // 128), dtype=np.int32)
    lib().orc_quant_w_128x128_pow2(_p(w), rows, cols, _p(q), _p(e))
    return q, e


def pow2_scales(e: np.ndarray) -> np.ndarray:
    """2^e as float64 (exact)."""
    return np.ldexp(1.0, np.asarray(e, dtype=np.int32))


# ------------------------------------------------------ redundant experts
# The pages name redundant experts for inference load balance (the 618zxw.cn
# news article) without an algorithm.  Reading: copies are given so as to
# minimise the largest number of rows one copy serves, max_e ceil(c_e/r_e),
# each extra copy to the expert whose copies currently serve the most rows
# (ties to the lower expert); an expert's rows (in token order) are cut into
# r_e consecutive pieces whose sizes differ by at most one, longer first.

def redundant_plan(counts, n_extra: int):
    """-> replicas [N] (copies per expert), slot_expert [N + n_extra]."""
    c = [int(v) for v in counts]
    rep = [1] * len(c)
    for _ in range(int(n_extra)):
        loads = [-(-c[e] // rep[e]) for e in range(len(c))]  # ceil
        best = max(range(len(c)), key=lambda e: (loads[e], -e))
        rep[best] += 1
    slots = [e for e in range(len(c)) for _ in range(rep[e])]
    return np.array(rep, np.int32), np.array(slots, np.int32)


def split_groups(expert_offsets, replicas):
    """Group table of the copies: (slot_offsets [S + 2], slot_weight [S + 1])
    for S = sum(replicas) slots; the last group is the shared expert's."""
    off = [int(v) for v in expert_offsets]
    N = len(replicas)
    starts, weights = [], []
    for e in range(N):
        c, r = off[e + 1] - off[e], int(replicas[e])
        q, extra = divmod(c, r)
        for j in range(r):
            starts.append(off[e] + j * q + min(j, extra))
            weights.append(e)
    starts += [off[N], off[N + 1]]
    weights.append(N)
    return np.array(starts, np.int32), np.array(weights, np.int32)


_TABLE = None


def _table():
    global _TABLE
    if _TABLE is None:
        _TABLE = e4m3_decode_table()
    return _TABLE


_POOL = None


def _row_pieces(rows: int, step: int, fill) -> None:
    """Run fill(r0, r1) over row ranges [r0, r1) of `step` rows (a multiple
    of the block height) on a thread pool.  Each element is written once by
    the same formula whatever the split: this only spreads the work over
    the host cores."""
    global _POOL
    if rows <= step:
        fill(0, rows)
        return
    if _POOL is None:
        from concurrent.futures import ThreadPoolExecutor
        _POOL = ThreadPoolExecutor(max(1, min(16, os.cpu_count() or 1)))
    list(_POOL.map(lambda r0: fill(r0, min(rows, r0 + step)), range(0, rows, step)))


def dequant_act(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """code value * tile scale, in FP64 (exact)."""
    rows, cols = q.shape
    out = np.empty((rows, cols), dtype=np.float64)

    def fill(r0, r1):
        v = _table()[q[r0:r1]].reshape(r1 - r0, cols // 128, 128)
        out[r0:r1] = (v * s[r0:r1].astype(np.float64)[:, :, None]).reshape(r1 - r0, cols)
    _row_pieces(rows, 256, fill)
    return out


def dequant_w(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """code value * block scale, in FP64 (exact)."""
    rows, cols = q.shape
    out = np.empty((rows, cols), dtype=np.float64)

    def fill(r0, r1):
        v = _table()[q[r0:r1]].reshape((r1 - r0) // 128, 128, cols // 128, 128)
        sb = s[r0 // 128:r1 // 128].astype(np.float64)
        out[r0:r1] = (v * sb[:, None, :, None]).reshape(r1 - r0, cols)
    _row_pieces(rows, 256, fill)
    return out


# ----------------------------------------------------------------- routing
def route(x_bf16: np.ndarray, router_w_bf16: np.ndarray, bias: np.ndarray,
          n_groups: int, topk_groups: int, topk: int,
          logit_offset: Optional[np.ndarray] = None, want_scores: bool = False) -> dict:
    T, d = x_bf16.shape
    n_routed = router_w_bf16.shape[0]
    x = _c(x_bf16, np.uint16)
    E = _c(router_w_bf16, np.uint16)
    b = _c(bias, np.float32)
    off = None if logit_offset is None else _c(logit_offset, np.float32)
    idx = np.empty((T, topk), dtype=np.int32)
    gate = np.empty((T, topk), dtype=np.float32)
    counts = np.empty((n_routed,), dtype=np.int32)
    logits = np.empty((T, n_routed), dtype=np.float32) if want_scores else None
    scores = np.empty((T, n_routed), dtype=np.float32) if want_scores else None
    rc = lib().orc_route(T, d, n_routed, n_groups, topk_groups, topk, _p(x), _p(E),
                         _p(b), _p(off), _p(idx), _p(gate), _p(counts), _p(logits),
                         _p(scores))
    if rc != 0:
        raise ValueError("invalid routing shape")
    out = {"topk_idx": idx, "topk_gate": gate, "counts": counts}
    if want_scores:
        out["logits"] = logits
        out["scores"] = scores
    return out


def update_bias(counts: np.ndarray, bias: np.ndarray, T: int, topk: int,
                gamma: float) -> np.ndarray:
    b = _c(bias, np.float32).copy()
    c = _c(counts, np.int32)
    lib().orc_update_bias(T, b.size, topk, _p(c), ctypes.c_float(gamma), _p(b))
    return b


def permute_layout(topk_idx: np.ndarray, counts: np.ndarray, n_routed: int):
    T, K = topk_idx.shape
    idx = _c(topk_idx, np.int32)
    c = _c(counts, np.int32)
    offsets = np.empty((n_routed + 2,), dtype=np.int32)
    rop = np.empty((T, K), dtype=np.int32)
    lib().orc_permute_layout(T, n_routed, K, _p(idx), _p(c), _p(offsets), _p(rop))
    return offsets, rop


# ----------------------------------------------------------------- experts
def quantized_expert(w1_bf16, w3_bf16, w2_bf16):
    """Oracle quantisation of one expert's bf16 weights (128x128 blocks)."""
    return quant_w_128x128(w1_bf16), quant_w_128x128(w3_bf16), quant_w_128x128(w2_bf16)


def quantized_expert_pow2(w1_bf16, w3_bf16, w2_bf16):
    """Oracle quantisation of one expert with power-of-two 128x128 scales;
    the scales are returned as float32 values 2^e (exact)."""
    out = []
    for w in (w1_bf16, w3_bf16, w2_bf16):
        q, e = quant_w_128x128_pow2(w)
        out.append((q, pow2_scales(e).astype(np.float32)))
    return tuple(out)


def quant_act_1x128_pow2_values(x: np.ndarray):
    """quant_act_1x128_pow2 with the scales as float32 values 2^e."""
    q, e = quant_act_1x128_pow2(x)
    return q, pow2_scales(e).astype(np.float32)


def swiglu_expert(xq: np.ndarray, xs: np.ndarray, w1, w3, w2,
                  return_h: bool = False, h_quant=None):
    """One expert on FP8 rows (xq, xs = 1x128 codes and scales).

    w1, w3, w2 = (codes, scales) pairs, [I,d], [I,d], [d,I].
    a = X W1^T and c = X W3^T in FP64 over dequantised values;
    h = silu(a) * c with silu(a) = a / (1 + exp(-a)), rounded to fp32;
    h re-quantised 1x128 along I (every Fprop GEMM input is FP8);
    o = H W2^T in FP64.  Returns o (FP64 [rows, d])."""
    X = dequant_act(xq, xs)
    W1 = dequant_w(*w1)
    W3 = dequant_w(*w3)
    a = X @ W1.T
    c = X @ W3.T
    h = (a / (1.0 + np.exp(-a))) * c
    h32 = h.astype(np.float32)
    hq, hs = (h_quant or quant_act_1x128)(h32)
    o = dequant_act(hq, hs) @ dequant_w(*w2).T
    if return_h:
        return o, h32, hq, hs
    return o


def f64_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round FP64 directly to bf16 (8 significant bits), nearest-even.

    Done in FP64: scale each value by a power of two so that the bf16 grid
    step is 1, rint (ties to even), scale back; all steps are exact.
    Values below the bf16 normal range use the subnormal step 2^-133."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    # correct floor(log2) at exact powers of two / rounding of log2
    e = np.where(np.ldexp(1.0, e.astype(np.int32)) > a, e - 1, e)
    e = np.where(np.ldexp(1.0, (e + 1).astype(np.int32)) <= a, e + 1, e)
    e = np.maximum(e, -126.0)
    step = np.ldexp(1.0, (e - 7).astype(np.int32))
    r = np.rint(a / step) * step
    r = np.where(a > 0, r, 0.0)
    r32 = np.copysign(r, v).astype(np.float32)  # exact: r is on the bf16 grid
    bits = r32.view(np.uint32) >> np.uint32(16)
    return bits.astype(np.uint16)


def combine(o_shared: np.ndarray, o_routed: np.ndarray, gates: np.ndarray) -> np.ndarray:
    """y_t = o_shared_t + sum_k g_tk * o_tk in FP64, rounded once to bf16.

    o_shared [T,d]; o_routed [T,K,d]; gates [T,K] fp32.  Returns bf16 bits."""
    y = o_shared + np.einsum("tk,tkd->td", gates.astype(np.float64), o_routed)
    return f64_to_bf16_bits(y)


def layer_forward(x_bf16: np.ndarray, router_w_bf16: np.ndarray, bias: np.ndarray,
                  n_groups: int, topk_groups: int, topk: int,
                  expert_weights: Callable[[int], tuple],
                  logit_offset: Optional[np.ndarray] = None,
                  tokens: Optional[np.ndarray] = None, scales: str = "fp32") -> dict:
    """Whole layer for all tokens (routing) and the chosen ``tokens`` (output).

    expert_weights(e) returns ((w1q,w1s),(w3q,w3s),(w2q,w2s)) for expert e;
    e = n_routed is the shared expert.  Experts are visited once each.
    Returns routing results, x codes/scales, and y (bf16 bits) for ``tokens``."""
    T, d = x_bf16.shape
    n_routed = router_w_bf16.shape[0]
    r = route(x_bf16, router_w_bf16, bias, n_groups, topk_groups, topk, logit_offset)
    # scales = "pow2": the power-of-two option for x and h (the expert
    # weights come quantised that way from expert_weights)
    act_quant = quant_act_1x128 if scales == "fp32" else quant_act_1x128_pow2_values
    xq, xs = act_quant(x_bf16)
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    idx = r["topk_idx"][tokens]
    gates = r["topk_gate"][tokens].astype(np.float64)
    # y_t = o_shared_t + sum_k g_tk o_tk in FP64, accumulated expert by
    # expert (a token meets each expert at most once), then one bf16 rounding
    y64 = np.zeros((len(tokens), d), dtype=np.float64)
    for e in range(n_routed + 1):
        if e == n_routed:
            sel = np.arange(len(tokens))
            slots = None
        else:
            sel, slots = np.nonzero(idx == e)
            if sel.size == 0:
                continue
        w = expert_weights(e)
        o = swiglu_expert(xq[tokens[sel]], xs[tokens[sel]], *w, h_quant=act_quant)
        if slots is None:
            y64[sel] += o
        else:
            y64[sel] += gates[sel, slots][:, None] * o
    y = f64_to_bf16_bits(y64)
    r.update({"xq": xq, "xs": xs, "y": y, "tokens": tokens})
    return r


def gemm_blockscaled(aq, a_s, bq, b_s):
    """C = dq(A) dq(B)^T in FP64; A [m,k] 1x128-scaled, B [n,k] 128x128-scaled."""
    return dequant_act(aq, a_s) @ dequant_w(bq, b_s).T


def gemm_wgrad(a_t, a_scales, b_t, b_scales, kb_offsets):
    """Weight-gradient GEMM with K groups: out[g] = dq(A)[:, K_g] dq(B)[:, K_g]^T
    in FP64, K_g the 128-column blocks [kb_offsets[g], kb_offsets[g+1]).
    a_t [m, nkb*128] codes with scales [nkb, m] (one per row and K block),
    b_t [n, nkb*128] likewise.  Returns [G, m, n]."""
    A = dequant_act(a_t, np.ascontiguousarray(a_scales.T))
    B = dequant_act(b_t, np.ascontiguousarray(b_scales.T))
    G = len(kb_offsets) - 1
    out = np.zeros((G, A.shape[0], B.shape[0]))
    for g in range(G):
        k0, k1 = 128 * int(kb_offsets[g]), 128 * int(kb_offsets[g + 1])
        out[g] = A[:, k0:k1] @ B[:, k0:k1].T
    return out


# ---------------------------------------------------------------- backward
# The gradient of the layer with respect to x and the router weights for an
# upstream gradient dy ("DeepSeek-V3 Technical Report" notes page, section
# "FP8 mixed precision training": the Fprop, Dgrad and Wgrad GEMMs run in
# FP8, gating stays in high precision; section "DeepSeekMoE and
# auxiliary-loss-free load balancing": gates are the normalised unbiased
# affinities of the selected experts, the bias only selects).  Readings:
#   - the selection is piecewise constant: no gradient flows through the
#     top-K choice or the bias;
#   - gates g_k = s_k / S with S the sum of the chosen s: dL/ds_j =
#     (dg_j - sum_k g_k dg_k) / S for chosen j; dL/du_j = dL/ds_j s_j (1-s_j);
#   - the expert MLP's Dgrad GEMMs take FP8 operands quantised like the
#     forward's: do = g dy (fp32 product) per routed row (dy for the shared
#     row) in 1x128 tiles along d, and [da | dc] in 1x128 tiles along 2I;
#     the weights keep their 128x128 blocks, transposed (exact);
#   - SwiGLU derivative: silu'(a) = sigma(a) (1 + a (1 - sigma(a))).

def gate_backward(dy_bf16: np.ndarray, o_routed: np.ndarray, scores: np.ndarray):
    """dg [T,K] = <dy_t, o_tk>, du [T,K] = dL/du of the chosen logits.
    o_routed: FP64 [T,K,d] routed expert outputs; scores: fp32 [T,K] the
    chosen experts' unbiased s."""
    dy = _bf16_to_f64(dy_bf16)
    dg = np.einsum("td,tkd->tk", dy, o_routed)
    s = scores.astype(np.float64)
    S = s.sum(axis=1, keepdims=True)
    g = s / S
    ds = (dg - (g * dg).sum(axis=1, keepdims=True)) / S
    du = ds * s * (1.0 - s)
    return dg, du


def router_backward(du: np.ndarray, topk_idx: np.ndarray, x_bf16: np.ndarray,
                    router_w_bf16: np.ndarray):
    """dx_router [T,d] = sum_k du_tk E_{e_k};  dE [N_r,d] = sum du_tk x_t."""
    x = _bf16_to_f64(x_bf16)
    E = _bf16_to_f64(router_w_bf16)
    dx = np.einsum("tk,tkd->td", du, E[topk_idx])
    dE = np.zeros_like(E)
    np.add.at(dE, topk_idx.ravel(), (du[:, :, None] * x[:, None, :]).reshape(-1, x.shape[1]))
    return dx, dE


def swiglu_backward(dh, a, c):
    """h = silu(a) c:  da = dh c silu'(a) with silu'(a) = sigma(a) (1 + a (1 -
    sigma(a))), dc = dh silu(a); FP64."""
    a = np.asarray(a, np.float64)
    sig = 1.0 / (1.0 + np.exp(-a))
    da = np.asarray(dh, np.float64) * np.asarray(c, np.float64) * sig * (1.0 + a * (1.0 - sig))
    dc = np.asarray(dh, np.float64) * a * sig
    return da, dc


def quant_act_128x1(x: np.ndarray):
    """128x1 tiles along the rows: a [rows, cols] matrix (one expert's rows)
    is cut into blocks of 128 rows from its first row, and every column of a
    block takes its own scale (the 1x128 rule applied to the transpose, the
    rows padded with zeros to a multiple of 128).  x: uint16 bf16 bits or
    float32.  Returns (codes uint8 [cols, rows_pad], scales float32
    [cols, rows_pad/128]): the transposed operand of a weight-gradient GEMM."""
    rows, cols = x.shape
    pad = -(-rows // 128) * 128
    t = np.zeros((cols, pad), dtype=x.dtype)
    t[:, :rows] = x.T
    return quant_act_1x128(t)


def expert_backward(do_rows_f32: np.ndarray, xq: np.ndarray, xs: np.ndarray, w1, w3, w2,
                    quant: bool = True, x_rows=None):
    """Dgrad through one expert for its rows: do (fp32 [rows, d], the
    gate-scaled dy) quantised 1x128 -> dh = dq(do) W2 (FP64); a, c
    recomputed from the forward's FP8 x; da = dh c silu'(a), dc = dh silu(a)
    rounded to fp32 and quantised 1x128 along [da | dc]; dx = dq([da|dc])
    [W1; W3] (FP64).  Returns dx [rows, d] FP64.
    quant=False (for checks against derivatives): no quantisation of do and
    [da | dc], and xq is taken as the FP64 input itself (xs ignored).

    With x_rows (the rows' layer input: bf16 bits, or FP64 when quant=False)
    also the weight gradients, contracting over the rows: returns (dx,
    dW13 [2I, d] = [da | dc]^T x, dW2 [d, I] = do^T h) with h = silu(a) c.
    Each operand is quantised in 128x1 tiles along the rows from its fp32
    value (do; h and [da | dc] rounded to fp32; x from bf16)."""
    W1, W3, W2 = dequant_w(*w1), dequant_w(*w3), dequant_w(*w2)
    if quant:
        dq_, ds_ = quant_act_1x128(np.ascontiguousarray(do_rows_f32, np.float32))
        dh = dequant_act(dq_, ds_) @ W2
        X = dequant_act(xq, xs)
    else:
        dh = np.asarray(do_rows_f32, np.float64) @ W2
        X = np.asarray(xq, np.float64)
    a, c = X @ W1.T, X @ W3.T
    dac_exact = np.concatenate(swiglu_backward(dh, a, c), axis=1)
    if quant:
        qq, qs = quant_act_1x128(dac_exact.astype(np.float32))
        dac = dequant_act(qq, qs)
    else:
        dac = dac_exact
    dx = dac @ np.concatenate([W1, W3], axis=0)
    if x_rows is None:
        return dx
    h = a / (1.0 + np.exp(-a)) * c
    if quant:
        rows = X.shape[0]

        def t128(m):  # dequantised transposed 128x1 operand, [cols, rows]
            q_, s_ = quant_act_128x1(m)
            return dequant_act(q_, s_)[:, :rows]
        dW2 = t128(np.ascontiguousarray(do_rows_f32, np.float32)) @ \
            t128(h.astype(np.float32)).T
        dW13 = t128(dac_exact.astype(np.float32)) @ \
            t128(np.ascontiguousarray(x_rows, np.uint16)).T
    else:
        dW2 = np.asarray(do_rows_f32, np.float64).T @ h
        dW13 = dac_exact.T @ np.asarray(x_rows, np.float64)
    return dx, dW13, dW2


def _bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def layer_backward(dy_bf16, x_bf16, router_w_bf16, bias, n_groups, topk_groups, topk,
                   expert_weights, logit_offset=None, quant=True, wgrad_experts=()):
    """dx [T,d] (FP64) and dE [N_r,d] (FP64) of the whole layer for dy.
    quant=False (for checks against derivatives): the experts take x itself
    and nothing is quantised (the routing is the same).
    wgrad_experts: experts (N_r = the shared one) whose weight gradients to
    return as "dW" {e: (dW13 [2I, d], dW2 [d, I])} (zeros for an expert no
    token chose)."""
    T, d = x_bf16.shape
    n_routed = router_w_bf16.shape[0]
    r = route(x_bf16, router_w_bf16, bias, n_groups, topk_groups, topk, logit_offset,
              want_scores=True)
    idx = r["topk_idx"]
    scores = np.take_along_axis(r["scores"], idx, axis=1)
    xq, xs = quant_act_1x128(x_bf16)
    dy32 = _bf16_to_f64(dy_bf16).astype(np.float32)
    gates = r["topk_gate"]
    o_routed = np.zeros((T, topk, d))
    dx = np.zeros((T, d))
    dW = {}
    for e in range(n_routed + 1):
        if e == n_routed:
            sel, slots = np.arange(T), None
            do = dy32
        else:
            sel, slots = np.nonzero(idx == e)
            if sel.size == 0:
                continue
            do = (gates[sel, slots].astype(np.float32)[:, None] * dy32[sel]).astype(np.float32)
        w = expert_weights(e)
        want_w = e in wgrad_experts
        if quant:
            if slots is not None:
                o_routed[sel, slots] = swiglu_expert(xq[sel], xs[sel], *w)
            res = expert_backward(do, xq[sel], xs[sel], *w,
                                  x_rows=x_bf16[sel] if want_w else None)
        else:
            X = _bf16_to_f64(x_bf16[sel])
            if slots is not None:
                W1, W3, W2 = (dequant_w(*m) for m in w)
                a, c = X @ W1.T, X @ W3.T
                o_routed[sel, slots] = (a / (1.0 + np.exp(-a)) * c) @ W2.T
            res = expert_backward(do, X, None, *w, quant=False, x_rows=X if want_w else None)
        if want_w:
            dx[sel] += res[0]
            dW[e] = (res[1], res[2])
        else:
            dx[sel] += res
    for e in wgrad_experts:
        if e not in dW:
            I2, dd = expert_weights(e)[0][0].shape
            dW[e] = (np.zeros((2 * I2, dd)), np.zeros((dd, I2)))
    dg, du = gate_backward(dy_bf16, o_routed, scores)
    dxr, dE = router_backward(du, idx, x_bf16, router_w_bf16)
    return {"dx": dx + dxr, "dE": dE, "dg": dg, "du": du, "topk_idx": idx, "scores": scores,
            "dW": dW}
