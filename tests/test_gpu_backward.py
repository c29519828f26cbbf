"""Backward pass on the GPU (through the C ABI) against the oracle
("DeepSeek-V3 Technical Report" notes page, section "FP8 mixed precision
training": Dgrad with FP8 operands, 1x128 tiles for activation gradients,
128x128 blocks for weights; section "DeepSeekMoE and auxiliary-loss-free
load balancing": gates from the chosen unbiased affinities, no gradient
through the choice or the bias).

Kernel by kernel on seeded synthetic inputs (the transposed weights and the
quantised output gradients bit-exact, the FP32 sums within their rounding
bounds), then the whole layer's dx and router gradient at the small shape
(all tokens, ragged batches) and at the full expert shapes (d = 7168,
I = 2048: 16 and 256 routed experts, all tokens)."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from gpu_util import (DEV, OracleExperts, bf16_dev, expert_bf16, need_gpu,
                      rel_frobenius, shape_of, to_dev)

pytestmark = pytest.mark.gpu

U32 = np.uint32


def _moe():
    import fp8_block_scaled_affinity_b200 as moe
    return moe


def _routing(rng, T, N, K, n_choosable=None):
    """Random distinct experts per token (from the first n_choosable), the
    counts and the oracle's permutation layout."""
    n_c = N if n_choosable is None else n_choosable
    idx = np.zeros((T, K), np.int32)
    for t in range(T):
        idx[t] = rng.permutation(n_c)[:K]
    counts = np.bincount(idx.ravel(), minlength=N).astype(np.int32)
    off, rop = oracle.permute_layout(idx, counts, N)
    return idx, counts, off, rop


def _report(rec):
    print(json.dumps(rec))
    path = os.environ.get("MOEFP8_PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(rec) + "\n")


# ------------------------------------------------------------- kernels
@pytest.mark.parametrize("mats,rows,cols", [(3, 256, 384), (1, 128, 128), (2, 640, 256),
                                            (0, 128, 128)])
def test_transpose_w_bit_exact(mats, rows, cols):
    need_gpu()
    rng = np.random.default_rng(10 + rows)
    q = rng.integers(0, 256, (mats, rows, cols), dtype=np.uint8)
    s = rng.random((mats, rows // 128, cols // 128)).astype(np.float32)
    qt = torch.full((mats, cols, rows), 7, dtype=torch.uint8, device=DEV)
    st = torch.zeros((mats, cols // 128, rows // 128), dtype=torch.float32, device=DEV)
    _moe().fp8_transpose_w_128x128(to_dev(q), to_dev(s), qt, st)
    torch.cuda.synchronize()
    assert np.array_equal(qt.cpu().numpy(), q.transpose(0, 2, 1))
    assert np.array_equal(st.cpu().numpy().view(U32), s.transpose(0, 2, 1).view(U32))


@pytest.mark.parametrize("T,d", [(37, 512), (5, 1792), (130, 7168)])
def test_combine_backward_quant_bit_exact(T, d):
    """do rows = fp32(gate * dy) (dy itself on the shared rows), quantised in
    1x128 tiles with the forward's rule, in the permutation's row order;
    d = 1792 and 7168 take the seven-vector piece form."""
    need_gpu()
    moe = _moe()
    N, G, M, K = 16, 4, 2, 4
    rng = np.random.default_rng(20 + d)
    dy = S.host_normal_bf16(rng, (T, d), 1.0)
    gate = rng.random((T, K)).astype(np.float32)
    idx, counts, off, rop = _routing(rng, T, N, K)
    R = T * K + T
    sh = moe.make_shape(T, d, N, G, M, K, 256)
    do_q = torch.zeros((R, d), dtype=torch.uint8, device=DEV)
    do_s = torch.zeros((d // 128, R), dtype=torch.float32, device=DEV)
    moe.moe_combine_backward_quant(sh, bf16_dev(dy), to_dev(rop), to_dev(gate), do_q, do_s)
    torch.cuda.synchronize()
    dy32 = S.bf16_bits_to_f32(dy)
    do32 = (gate[:, :, None] * dy32[:, None, :]).astype(np.float32).reshape(T * K, d)
    q_pairs, s_pairs = oracle.quant_act_1x128(do32)
    q_sh, s_sh = oracle.quant_act_1x128(np.ascontiguousarray(dy32))
    exp_q = np.zeros((R, d), np.uint8)
    exp_s = np.zeros((R, d // 128), np.float32)
    exp_q[rop.ravel()] = q_pairs
    exp_s[rop.ravel()] = s_pairs
    exp_q[T * K:] = q_sh
    exp_s[T * K:] = s_sh
    assert np.array_equal(do_q.cpu().numpy(), exp_q)
    assert np.array_equal(do_s.cpu().numpy().T.view(U32), exp_s.view(U32))


@pytest.mark.parametrize("rows,inter", [(300, 256), (77, 896), (130, 2048)])
def test_swiglu_backward_quant(rows, inter):
    """[da | dc] from fp32 dh and [a | c]: the GPU's fp32 arithmetic against
    the FP64 definition.  Codes equal the oracle's quantisation of the FP64
    values rounded to fp32 except where the few-ulp fp32 difference crosses
    an E4M3 rounding boundary; every dequantised value is within one E4M3
    step of the exact gradient."""
    need_gpu()
    moe = _moe()
    rng = np.random.default_rng(30 + inter)
    dh = rng.standard_normal((rows, inter)).astype(np.float32)
    ac = (rng.standard_normal((rows, 2 * inter)) * 2.0).astype(np.float32)
    q = torch.zeros((rows, 2 * inter), dtype=torch.uint8, device=DEV)
    qs = torch.zeros((2 * inter // 128, rows), dtype=torch.float32, device=DEV)
    moe.moe_swiglu_backward_quant(to_dev(dh), to_dev(ac), rows, inter, rows, q, qs)
    torch.cuda.synchronize()
    da, dc = oracle.swiglu_backward(dh, ac[:, :inter], ac[:, inter:])
    exact = np.concatenate([da, dc], axis=1)
    q_ref, s_ref = oracle.quant_act_1x128(exact.astype(np.float32))
    q_got, s_got = q.cpu().numpy(), qs.cpu().numpy().T.copy()
    assert np.all(np.abs(s_got - s_ref) <= 16 * 2.0**-24 * np.abs(s_ref))
    same = float(np.mean(q_got == q_ref))
    deq = oracle.dequant_act(q_got, s_got)
    step = np.repeat(s_got, 128, axis=1)
    assert np.all(np.abs(deq - exact) <= 2.0**-3 * np.abs(exact) + 2.0**-9 * step)
    _report({"case": f"swiglu backward quant {rows}x{2 * inter}", "codes_equal_frac": same})
    assert same >= 0.999


def test_gate_backward():
    need_gpu()
    moe = _moe()
    T, d, N, G, M, K = 50, 512, 64, 8, 4, 8
    rng = np.random.default_rng(40)
    dy = S.host_normal_bf16(rng, (T, d), 1.0)
    idx, counts, off, rop = _routing(rng, T, N, K)
    R = T * K + T
    o = rng.standard_normal((R, d)).astype(np.float32)
    score = (0.05 + 0.9 * rng.random((T, K))).astype(np.float32)
    sh = moe.make_shape(T, d, N, G, M, K, 256)
    dg = torch.empty((T, K), dtype=torch.float32, device=DEV)
    du = torch.empty((T, K), dtype=torch.float32, device=DEV)
    moe.moe_gate_backward(sh, bf16_dev(dy), to_dev(o), to_dev(rop), to_dev(score), dg, du)
    torch.cuda.synchronize()
    dg_ref, du_ref = oracle.gate_backward(dy, o[rop].astype(np.float64), score)
    # both sides sum in FP64 (different order) and round once to fp32
    mag = np.einsum("td,tkd->tk", np.abs(S.bf16_bits_to_f32(dy).astype(np.float64)),
                    np.abs(o[rop].astype(np.float64)))
    assert np.all(np.abs(dg.cpu().numpy() - dg_ref) <= 2.0**-24 * np.abs(dg_ref) + 1e-13 * mag)
    du_mag = mag.sum(axis=1, keepdims=True) / score.sum(axis=1, keepdims=True)
    assert np.all(np.abs(du.cpu().numpy() - du_ref) <= 2.0**-24 * np.abs(du_ref) + 1e-13 * du_mag)


@pytest.mark.parametrize("T,N", [(70, 32), (600, 8)])
def test_router_backward(T, N):
    """dx_router and dE (fp32 sums) within their rounding bounds; an expert
    no token chose gets an exact zero row; at T = 600 each expert's rows
    span several 128-row blocks (partial sums added in order)."""
    need_gpu()
    moe = _moe()
    d, G, M, K = 512, 4, 2, 4
    rng = np.random.default_rng(50)
    x = S.host_normal_bf16(rng, (T, d), 1.0)
    E = S.host_normal_bf16(rng, (N, d), 0.02)
    du = rng.standard_normal((T, K)).astype(np.float32)
    idx, counts, off, rop = _routing(rng, T, N, K, n_choosable=N - 1)
    sh = moe.make_shape(T, d, N, G, M, K, 256)
    dxr = torch.empty((T, d), dtype=torch.float32, device=DEV)
    dE = torch.full((N, d), 5.0, dtype=torch.float32, device=DEV)
    scratch = torch.empty((T * K,), dtype=torch.int32, device=DEV)
    st = torch.zeros((1,), dtype=torch.int32, device=DEV)
    ws = torch.empty((moe.moe_router_backward_workspace_size(sh),), dtype=torch.uint8,
                     device=DEV)
    moe.moe_router_backward(sh, bf16_dev(x), bf16_dev(E), to_dev(du), to_dev(idx), to_dev(off),
                            to_dev(rop), scratch, dxr, dE, ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    dx_ref, dE_ref = oracle.router_backward(du.astype(np.float64), idx, x, E)
    bx, bE = oracle.router_backward(np.abs(du.astype(np.float64)), idx, x & 0x7FFF, E & 0x7FFF)
    assert np.all(np.abs(dxr.cpu().numpy() - dx_ref) <= (K + 1) * 2.0**-23 * bx)
    cmax = int(counts.max())
    assert np.all(np.abs(dE.cpu().numpy() - dE_ref) <= (cmax + 1) * 2.0**-23 * bE)
    assert np.all(dE.cpu().numpy()[N - 1] == 0.0)


@pytest.mark.parametrize("with_router", [True, False])
def test_dx_combine(with_router):
    need_gpu()
    moe = _moe()
    T, d, N, G, M, K = 33, 512, 16, 4, 2, 4
    rng = np.random.default_rng(60)
    idx, counts, off, rop = _routing(rng, T, N, K)
    R = T * K + T
    rows = rng.standard_normal((R, d)).astype(np.float32)
    dxr = rng.standard_normal((T, d)).astype(np.float32)
    sh = moe.make_shape(T, d, N, G, M, K, 256)
    dx = torch.empty((T, d), dtype=torch.float32, device=DEV)
    moe.moe_dx_combine(sh, to_dev(rows), to_dev(dxr) if with_router else None, to_dev(rop), dx)
    torch.cuda.synchronize()
    r64 = rows.astype(np.float64)
    ref = r64[T * K:] + r64[rop].sum(axis=1)
    mag = np.abs(r64[T * K:]) + np.abs(r64[rop]).sum(axis=1)
    if with_router:
        ref += dxr
        mag += np.abs(dxr)
    assert np.all(np.abs(dx.cpu().numpy() - ref) <= (K + 2) * 2.0**-24 * mag)


# ----------------------------------------------------------- the layer
# dx: the expert chain is FP8 on both sides with the same quantisation points;
# the GPU's FP32 sums against the oracle's FP64 move a [da|dc] code by one E4M3
# step only where the difference crosses a rounding boundary.  The router part
# (du) depends on the expert outputs o, whose h codes differ in the same rare
# way as in the forward (a token's y is off by up to about a percent there).
DX_TOL, DX_TOKEN_TOL, DE_TOL = 2e-3, 5e-2, 2e-2


def _layer_case(name, cfg, T=None, seed=70):
    need_gpu()
    moe = _moe()
    inp = S.make_layer_inputs_host(cfg, 0)
    T = cfg.T if T is None else T
    layer = moe.MoeLayer(shape_of(cfg, T), bf16_dev(inp["router_w"]), to_dev(inp["bias"]),
                         device=DEV)
    for e in range(cfg.n_routed + 1):
        layer.set_expert(e, *expert_bf16(cfg, e))
    x = inp["x"][:T]
    off = inp["logit_offset"]
    xd = bf16_dev(x)
    y_train = layer.forward_train(xd, logit_offset=None if off is None else to_dev(off))
    y_fwd = layer.forward(xd, logit_offset=None if off is None else to_dev(off))
    torch.cuda.synchronize()
    assert torch.equal(y_train.view(torch.int16), y_fwd.view(torch.int16))
    dy = S.host_normal_bf16(np.random.default_rng(seed), (T, cfg.d), 1.0)
    dx, dE = layer.backward(bf16_dev(dy))
    torch.cuda.synchronize()
    assert layer.status() == 0
    ref = oracle.layer_backward(dy, x, inp["router_w"], inp["bias"], cfg.n_groups,
                                cfg.topk_groups, cfg.topk, OracleExperts(cfg), logit_offset=off)
    assert np.array_equal(layer.topk_idx.cpu().numpy(), ref["topk_idx"])
    got = dx.cpu().numpy().astype(np.float64)
    fro = rel_frobenius(got, ref["dx"])
    tok = (np.linalg.norm(got - ref["dx"], axis=1) /
           np.maximum(np.linalg.norm(ref["dx"], axis=1), 1e-30))
    rec = {"case": f"backward {name}: {T} tokens", "dx_rel_frobenius": fro,
           "dx_worst_token_rel": float(tok.max()) if T else 0.0,
           "dE_rel_frobenius": rel_frobenius(dE.cpu().numpy(), ref["dE"]),
           "du_rel_frobenius": rel_frobenius(layer.last_du.cpu().numpy(), ref["du"])}
    _report(rec)
    assert fro <= DX_TOL, rec
    assert T == 0 or tok.max() <= DX_TOKEN_TOL, rec
    assert rec["dE_rel_frobenius"] <= DE_TOL, rec
    return rec


def test_layer_backward_tiny_all_tokens():
    _layer_case("tiny", S.CONFIGS["tiny"])


@pytest.mark.parametrize("T", [1, 13])
def test_layer_backward_tiny_ragged(T):
    _layer_case("tiny", S.CONFIGS["tiny"], T=T)


def test_layer_backward_full_expert_shapes_16_experts():
    _layer_case("prefill_e16", S.CONFIGS["prefill_e16"])


def test_layer_backward_decode_full_size():
    _layer_case("decode", S.CONFIGS["decode"])


# ------------------------------------------------------ weight gradients
def _inverse(rop, R):
    """pair_of_row of the routed rows from row_of_pair (host)."""
    inv = np.zeros((rop.size,), np.int32)
    inv[rop.ravel()] = np.arange(rop.size, dtype=np.int32)
    return inv


def _layout_ref(off, max_blocks):
    G = len(off) - 1
    kb = np.zeros(G + 1, np.int32)
    blocks = np.zeros((max_blocks, 2), np.int32)
    for g in range(G):
        rows = int(off[g + 1] - off[g])
        nb = -(-rows // 128)
        kb[g + 1] = kb[g] + nb
        for j in range(nb):
            blocks[kb[g] + j] = (off[g] + 128 * j, min(128, rows - 128 * j))
    return kb, blocks


def test_wgrad_layout_bit_exact():
    need_gpu()
    moe = _moe()
    sizes = [0, 1, 127, 128, 129, 0, 300, 5, 0]
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    nb = moe.moe_wgrad_max_blocks(off[-1], len(sizes))
    kb = torch.empty((len(sizes) + 1,), dtype=torch.int32, device=DEV)
    blocks = torch.full((nb, 2), 9, dtype=torch.int32, device=DEV)
    moe.moe_wgrad_layout(len(sizes), to_dev(off), kb, blocks)
    torch.cuda.synchronize()
    kb_ref, blocks_ref = _layout_ref(off, nb)
    assert np.array_equal(kb.cpu().numpy(), kb_ref)
    assert np.array_equal(blocks.cpu().numpy(), blocks_ref)


def _wgrad_setup(T, d, N, K, seed):
    rng = np.random.default_rng(seed)
    idx, counts, off, rop = _routing(rng, T, N, K, n_choosable=N - 1)
    R = T * K + T
    moe = _moe()
    nb = moe.moe_wgrad_max_blocks(R, N + 1)
    kb = torch.empty((N + 2,), dtype=torch.int32, device=DEV)
    blocks = torch.empty((nb, 2), dtype=torch.int32, device=DEV)
    moe.moe_wgrad_layout(N + 1, to_dev(off), kb, blocks)
    torch.cuda.synchronize()
    return rng, idx, off, rop, R, nb, kb, blocks


def _expert_rows(off, e):
    return np.arange(off[e], off[e + 1])


@pytest.mark.parametrize("source", ["x", "do"])
def test_wgrad_quant_x_and_do_bit_exact(source):
    """The transposed 128x1 operands of x and of do = fp32(gate dy) equal the
    oracle's 128x1 quantisation of each expert's rows (in permutation order),
    codes and scales; an unchosen expert has no blocks."""
    need_gpu()
    moe = _moe()
    T, d, N, G, M, K = 150, 256, 8, 2, 2, 2
    rng, idx, off, rop, R, nb, kb, blocks = _wgrad_setup(T, d, N, K, 80)
    x = S.host_normal_bf16(rng, (T, d), 1.0)
    gate = rng.random((T, K)).astype(np.float32)
    inv = _inverse(rop, R)
    sh = moe.make_shape(T, d, N, G, M, K, 128)
    q = torch.zeros((d, nb * 128), dtype=torch.uint8, device=DEV)
    s = torch.zeros((nb, d), dtype=torch.float32, device=DEV)
    if source == "x":
        moe.moe_wgrad_quant_x(sh, bf16_dev(x), to_dev(inv), blocks, q, s)
    else:
        moe.moe_wgrad_quant_do(sh, bf16_dev(x), to_dev(gate), to_dev(inv), blocks, q, s)
    torch.cuda.synchronize()
    q, s, kbh = q.cpu().numpy(), s.cpu().numpy(), kb.cpu().numpy()
    x32 = S.bf16_bits_to_f32(x)
    for e in range(N + 1):
        rows = _expert_rows(off, e)
        if rows.size == 0:
            assert kbh[e] == kbh[e + 1]
            continue
        toks = np.where(rows >= T * K, rows - T * K, inv[np.minimum(rows, T * K - 1)] // K)
        if source == "x":
            vals = x[toks]
        else:
            g = np.where(rows >= T * K, np.float32(1.0),
                         gate.ravel()[inv[np.minimum(rows, T * K - 1)]]).astype(np.float32)
            vals = (g[:, None] * x32[toks]).astype(np.float32)
        q_ref, s_ref = oracle.quant_act_128x1(np.ascontiguousarray(vals))
        k0, k1 = int(kbh[e]), int(kbh[e + 1])
        assert np.array_equal(q[:, 128 * k0:128 * k1], q_ref), e
        assert np.array_equal(s[k0:k1].T.view(U32), s_ref.view(U32)), e


@pytest.mark.parametrize("source", ["h", "dac"])
def test_wgrad_quant_h_and_dac(source):
    """h = silu(a) c and [da | dc] from fp32 inputs: codes equal the oracle's
    quantisation of the FP64 values (rounded to fp32) except at rare E4M3
    rounding boundaries; dequantised within one step of the exact value."""
    need_gpu()
    moe = _moe()
    T, d, N, K, I = 150, 256, 8, 2, 256
    rng, idx, off, rop, R, nb, kb, blocks = _wgrad_setup(T, d, N, K, 81)
    ac = (rng.standard_normal((R, 2 * I)) * 2.0).astype(np.float32)
    dh = rng.standard_normal((R, I)).astype(np.float32)
    F = I if source == "h" else 2 * I
    q = torch.zeros((F, nb * 128), dtype=torch.uint8, device=DEV)
    s = torch.zeros((nb, F), dtype=torch.float32, device=DEV)
    if source == "h":
        moe.moe_wgrad_quant_h(to_dev(ac), I, blocks, q, s)
    else:
        moe.moe_wgrad_quant_dac(to_dev(dh), to_dev(ac), I, blocks, q, s)
    torch.cuda.synchronize()
    q, s, kbh = q.cpu().numpy(), s.cpu().numpy(), kb.cpu().numpy()
    a64, c64 = ac[:, :I].astype(np.float64), ac[:, I:].astype(np.float64)
    if source == "h":
        exact = a64 / (1.0 + np.exp(-a64)) * c64
    else:
        exact = np.concatenate(oracle.swiglu_backward(dh, a64, c64), axis=1)
    same, total = 0, 0
    for e in range(N + 1):
        rows = _expert_rows(off, e)
        if rows.size == 0:
            continue
        k0, k1 = int(kbh[e]), int(kbh[e + 1])
        q_ref, s_ref = oracle.quant_act_128x1(exact[rows].astype(np.float32))
        qe, se = q[:, 128 * k0:128 * k1], s[k0:k1].T.copy()
        assert np.all(np.abs(se - s_ref) <= 16 * 2.0**-24 * np.abs(s_ref)), e
        same += int(np.sum(qe == q_ref))
        total += qe.size
        deq = oracle.dequant_act(qe, se)[:, :rows.size].T
        step = np.repeat(se.T, 128, axis=0)[:rows.size]
        ex = exact[rows]
        assert np.all(np.abs(deq - ex) <= 2.0**-3 * np.abs(ex) + 2.0**-9 * step), e
    _report({"case": f"wgrad quant {source}", "codes_equal_frac": same / total})
    assert same / total >= 0.999


@pytest.mark.parametrize("m,n,kbs", [(256, 512, [0, 3, 3, 5, 9]), (128, 256, [0, 1]),
                                     (384, 768, [0, 0, 2, 2, 20])])
def test_grouped_gemm_wgrad(m, n, kbs):
    """K-grouped GEMM with per-row scales on both operands against the
    oracle, within the FP32 accumulation bound; empty groups give zeros."""
    need_gpu()
    moe = _moe()
    rng = np.random.default_rng(90 + m)
    nkb = kbs[-1] + 1  # one trailing block no group uses
    table = oracle.e4m3_decode_table()
    finite = np.nonzero(np.isfinite(table))[0].astype(np.uint8)
    a = rng.choice(finite, (m, 128 * nkb)).astype(np.uint8)
    b = rng.choice(finite, (n, 128 * nkb)).astype(np.uint8)
    sa = (2.0 ** rng.uniform(-12, -6, (nkb, m))).astype(np.float32)
    sb = (2.0 ** rng.uniform(-12, -6, (nkb, n))).astype(np.float32)
    kb_off = np.array(kbs, np.int32)
    G = len(kbs) - 1
    out = torch.full((G, m, n), 3.0, dtype=torch.float32, device=DEV)
    st = torch.zeros((1,), dtype=torch.int32, device=DEV)
    moe.moe_grouped_gemm_wgrad(G, to_dev(kb_off), nkb, to_dev(a), to_dev(sa), m, to_dev(b),
                               to_dev(sb), n, out, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = oracle.gemm_wgrad(a, sa, b, sb, kb_off)
    # the same sums over |products|: codes with the sign bit cleared
    mag = oracle.gemm_wgrad((a & 0x7F).astype(np.uint8), sa, (b & 0x7F).astype(np.uint8), sb,
                            kb_off)
    got = out.cpu().numpy()
    nk = np.diff(kb_off)[:, None, None]
    assert np.all(np.abs(got - ref) <= 2.0**-23 * (128 + nk + 2) * mag)
    for g in range(G):
        if kb_off[g] == kb_off[g + 1]:
            assert np.all(got[g] == 0.0)


DW_TOL = 2e-3


def _wgrad_case(name, cfg, T=None, experts=None, seed=71):
    need_gpu()
    moe = _moe()
    inp = S.make_layer_inputs_host(cfg, 0)
    T = cfg.T if T is None else T
    layer = moe.MoeLayer(shape_of(cfg, T), bf16_dev(inp["router_w"]), to_dev(inp["bias"]),
                         device=DEV)
    for e in range(cfg.n_routed + 1):
        layer.set_expert(e, *expert_bf16(cfg, e))
    x = inp["x"][:T]
    off = inp["logit_offset"]
    layer.forward_train(bf16_dev(x), logit_offset=None if off is None else to_dev(off))
    dy = S.host_normal_bf16(np.random.default_rng(seed), (T, cfg.d), 1.0)
    dx, dE, dW13, dW2 = layer.backward(bf16_dev(dy), wgrad=True)
    torch.cuda.synchronize()
    assert layer.status() == 0
    counts = layer.expert_counts.cpu().numpy()
    if experts is None:
        experts = list(range(cfg.n_routed + 1))
    ref = oracle.layer_backward(dy, x, inp["router_w"], inp["bias"], cfg.n_groups,
                                cfg.topk_groups, cfg.topk, OracleExperts(cfg), logit_offset=off,
                                wgrad_experts=tuple(experts))
    worst = 0.0
    for e in experts:
        r13, r2 = ref["dW"][e]
        g13, g2 = dW13[e].cpu().numpy(), dW2[e].cpu().numpy()
        if e < cfg.n_routed and counts[e] == 0:
            assert not np.any(g13) and not np.any(g2), e
            continue
        err = max(rel_frobenius(g13, r13), rel_frobenius(g2, r2))
        worst = max(worst, err)
        assert err <= DW_TOL, (e, err)
    _report({"case": f"wgrad {name}: {T} tokens, {len(experts)} experts",
             "worst_dW_rel_frobenius": worst})


def test_layer_wgrad_tiny_all_experts():
    _wgrad_case("tiny", S.CONFIGS["tiny"])


def test_layer_wgrad_tiny_ragged():
    _wgrad_case("tiny", S.CONFIGS["tiny"], T=13)


def test_layer_wgrad_full_expert_shapes():
    """d = 7168, I = 2048, 16 routed experts: the shared expert and three
    routed ones (the oracle's FP64 weight gradients are 0.35 GB each)."""
    _wgrad_case("prefill_e16", S.CONFIGS["prefill_e16"], experts=[16, 0, 5, 11])


def test_layer_backward_empty_batch():
    """T = 0: every gradient is empty or zero (the weight gradients of every
    expert, the router's gradient), and nothing faults."""
    need_gpu()
    moe = _moe()
    cfg = S.CONFIGS["tiny"]
    inp = S.make_layer_inputs_host(cfg, 0)
    layer = moe.MoeLayer(shape_of(cfg, 0), bf16_dev(inp["router_w"]), to_dev(inp["bias"]),
                         device=DEV)
    for e in range(cfg.n_routed + 1):
        layer.set_expert(e, *expert_bf16(cfg, e))
    x = bf16_dev(inp["x"][:0])
    layer.forward_train(x)
    dx, dE, dW13, dW2 = layer.backward(bf16_dev(inp["x"][:0]), wgrad=True)
    torch.cuda.synchronize()
    assert layer.status() == 0
    assert dx.shape == (0, cfg.d)
    assert not torch.any(dE) and not torch.any(dW13) and not torch.any(dW2)
