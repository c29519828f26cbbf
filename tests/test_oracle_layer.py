"""Pins of the oracle's bias update, permutation layout, block-scaled GEMM,
SwiGLU expert, combine and bf16 output ("DeepSeek-V3 Technical Report" notes
page, sections "DeepSeekMoE and auxiliary-loss-free load balancing" and
"FP8 mixed precision training"; the combine is the "all-to-all combine" stage
of section "DualPipe", reduced to one GPU)."""
from fractions import Fraction

import numpy as np

import oracle
import synthetic as S
from conftest import read_golden
from exact import (bf16_bits_to_fraction, e4m3_from_bits, round_to_bf16_bits,
                   round_to_f32, silu_fraction)


def test_bias_update_hand_example():
    rows = {r[0]: r[1:] for r in read_golden("bias_update.txt")}
    counts = np.array([int(v) for v in rows["counts"]], np.int32)
    before = np.array([float(v) for v in rows["before"]], np.float32)
    after = np.array([float(v) for v in rows["after"]], np.float32)
    got = oracle.update_bias(counts, before, T=4, topk=2, gamma=0.125)
    assert np.array_equal(got, after)


def test_bias_update_directions_on_tiny_workload():
    cfg = S.CONFIGS["tiny"]
    inp = S.make_layer_inputs_host(cfg)
    r = oracle.route(inp["x"], inp["router_w"], inp["bias"], cfg.n_groups,
                     cfg.topk_groups, cfg.topk)
    b = oracle.update_bias(r["counts"], inp["bias"], cfg.T, cfg.topk, cfg.gamma)
    mean = cfg.T * cfg.topk / cfg.n_routed
    for i, c in enumerate(r["counts"]):
        if c > mean:
            assert b[i] < inp["bias"][i]
        elif c < mean:
            assert b[i] > inp["bias"][i]
        else:
            assert b[i] == inp["bias"][i]
        assert abs(float(b[i]) - float(inp["bias"][i])) <= cfg.gamma * (1 + 2 ** -20)


def test_permute_layout_is_stable_and_bijective():
    rng = np.random.default_rng(7)
    T, K, N = 300, 4, 16
    idx = np.stack([rng.choice(N, K, replace=False) for _ in range(T)]).astype(np.int32)
    counts = np.bincount(idx.ravel(), minlength=N).astype(np.int32)
    off, rop = oracle.permute_layout(idx, counts, N)
    assert off[0] == 0 and off[N] == T * K and off[N + 1] == T * K + T
    assert np.array_equal(np.diff(off[:N + 1]), counts)
    assert np.array_equal(np.sort(rop.ravel()), np.arange(T * K))
    for e in range(N):
        t, k = np.nonzero(idx == e)
        rows = rop[t, k]
        assert np.all((rows >= off[e]) & (rows < off[e + 1]))
        assert np.array_equal(rows[np.argsort(t)], np.arange(off[e], off[e + 1]))


def _exact_entry(aq, a_s, bq, b_s, i, j, val):
    """sum over K-blocks of sa*sb*sum(qa*qb) in exact rationals: a different
    formulation from the oracle's dequantise-then-matmul."""
    tot = Fraction(0)
    for kb in range(aq.shape[1] // 128):
        acc = sum(val[aq[i, kb * 128 + t]] * val[bq[j, kb * 128 + t]] for t in range(128))
        tot += acc * Fraction(float(a_s[i, kb])) * Fraction(float(b_s[j // 128, kb]))
    return tot


def test_blockscaled_gemm_against_exact_rationals():
    rng = np.random.default_rng(8)
    a = S.host_normal_bf16(rng, (3, 256), 1.0)
    b = S.host_normal_bf16(rng, (256, 256), 0.05)
    aq, a_s = oracle.quant_act_1x128(a)
    bq, b_s = oracle.quant_w_128x128(b)
    c = oracle.gemm_blockscaled(aq, a_s, bq, b_s)
    val = [e4m3_from_bits(cc) for cc in range(256)]
    for i in range(3):
        for j in (0, 1, 127, 128, 200, 255):
            tot = _exact_entry(aq, a_s, bq, b_s, i, j, val)
            assert abs(c[i, j] - float(tot)) <= 1e-13 * max(1.0, abs(float(tot)))


def test_silu_and_swiglu_by_hand():
    # silu(1) = 1/(1+e^-1) = 0.7310585786300049 (decimal, 16 digits)
    assert abs(float(silu_fraction(Fraction(1))) - 0.7310585786300049) < 1e-15
    assert silu_fraction(Fraction(0)) == 0
    # one expert, two tokens: check h against exact matmuls + decimal silu
    rng = np.random.default_rng(9)
    d, I = 128, 128
    x = S.host_normal_bf16(rng, (2, d), 1.0)
    w1 = S.host_normal_bf16(rng, (I, d), 0.05)
    w3 = S.host_normal_bf16(rng, (I, d), 0.05)
    w2 = S.host_normal_bf16(rng, (d, I), 0.05)
    xq, xs = oracle.quant_act_1x128(x)
    W = oracle.quantized_expert(w1, w3, w2)
    o, h32, hq, hs = oracle.swiglu_expert(xq, xs, *W, return_h=True)
    val = [e4m3_from_bits(cc) for cc in range(256)]
    for t in range(2):
        X = [val[c] * Fraction(float(xs[t, 0])) for c in xq[t]]
        for f in (0, 5, 77, 127):
            a = sum(X[k] * val[W[0][0][f, k]] for k in range(d)) * Fraction(float(W[0][1][0, 0]))
            c = sum(X[k] * val[W[1][0][f, k]] for k in range(d)) * Fraction(float(W[1][1][0, 0]))
            h = silu_fraction(a) * c
            assert h32[t, f] == round_to_f32(h)
        # o from the (separately pinned) quantised h, exactly
        H = [val[c] * Fraction(float(hs[t, 0])) for c in hq[t]]
        for j in (0, 64, 127):
            oe = sum(H[k] * val[W[2][0][j, k]] for k in range(I)) * Fraction(float(W[2][1][0, 0]))
            assert abs(o[t, j] - float(oe)) <= 1e-13 * max(1e-30, abs(float(oe)))


def test_bf16_rounding_hand_values():
    for val_s, bits_s in read_golden("bf16_round.txt"):
        got = int(oracle.f64_to_bf16_bits(np.array([float(val_s)]))[0])
        assert got == int(bits_s, 16), (val_s, hex(got))


def test_bf16_rounding_against_integer_rounding():
    rng = np.random.default_rng(10)
    v = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
                        1.0 + (rng.integers(0, 1 << 20, 2000) * 2.0 ** -28)])
    got = oracle.f64_to_bf16_bits(v)
    for i in range(0, v.size, 7):
        assert int(got[i]) == round_to_bf16_bits(Fraction(float(v[i]))), v[i]


def test_combine_sums_shared_and_gated_outputs():
    rng = np.random.default_rng(11)
    T, K, d = 5, 3, 16
    o_sh = rng.standard_normal((T, d))
    o_r = rng.standard_normal((T, K, d))
    g = rng.uniform(0, 1, (T, K)).astype(np.float32)
    y = oracle.combine(o_sh, o_r, g)
    for t in range(T):
        for j in range(d):
            exact = Fraction(float(o_sh[t, j])) + sum(Fraction(float(g[t, k])) *
                                                      Fraction(float(o_r[t, k, j]))
                                                      for k in range(K))
            assert int(y[t, j]) == round_to_bf16_bits(exact)


def test_layer_forward_tiny_consistency():
    """Whole-layer oracle on the tiny workload: every token's y equals the
    shared expert plus the gate-weighted selected experts, expert by expert."""
    cfg = S.CONFIGS["tiny"]
    inp = S.make_layer_inputs_host(cfg)
    W = {e: oracle.quantized_expert(*S.host_expert_weights(cfg, e))
         for e in range(cfg.n_routed + 1)}
    out = oracle.layer_forward(inp["x"], inp["router_w"], inp["bias"], cfg.n_groups,
                               cfg.topk_groups, cfg.topk, W.__getitem__)
    t = 17
    sel = out["topk_idx"][t]
    xq, xs = out["xq"][t:t + 1], out["xs"][t:t + 1]
    acc = oracle.swiglu_expert(xq, xs, *W[cfg.n_routed])[0].copy()
    for k, e in enumerate(sel):
        acc += float(out["topk_gate"][t, k]) * oracle.swiglu_expert(xq, xs, *W[int(e)])[0]
    assert np.array_equal(out["y"][t], oracle.f64_to_bf16_bits(acc))
    y = S.bf16_bits_to_f32(out["y"])
    assert np.isfinite(y).all() and np.abs(y).max() > 0


def test_layer_forward_pow2_option_recomposes():
    """The power-of-two scale option of the whole-layer oracle: a token's y is
    the shared expert plus the gate-weighted selected experts, with x, the
    weights and h quantised by the power-of-two rule (pinned in
    test_oracle_pow2.py) and the routing of the pages' recipe unchanged."""
    cfg = S.CONFIGS["tiny"]
    inp = S.make_layer_inputs_host(cfg)
    W = {e: oracle.quantized_expert_pow2(*S.host_expert_weights(cfg, e))
         for e in range(cfg.n_routed + 1)}
    out = oracle.layer_forward(inp["x"], inp["router_w"], inp["bias"], cfg.n_groups,
                               cfg.topk_groups, cfg.topk, W.__getitem__, scales="pow2")
    ref = oracle.route(inp["x"], inp["router_w"], inp["bias"], cfg.n_groups, cfg.topk_groups,
                       cfg.topk)
    assert np.array_equal(out["topk_idx"], ref["topk_idx"])
    qx, ex = oracle.quant_act_1x128_pow2(inp["x"])
    assert np.array_equal(out["xq"], qx)
    assert np.array_equal(out["xs"], np.ldexp(1.0, ex).astype(np.float32))
    t = 29
    xq, xs = out["xq"][t:t + 1], out["xs"][t:t + 1]
    hq = oracle.quant_act_1x128_pow2_values
    acc = oracle.swiglu_expert(xq, xs, *W[cfg.n_routed], h_quant=hq)[0].copy()
    for k, e in enumerate(out["topk_idx"][t]):
        acc += float(out["topk_gate"][t, k]) * oracle.swiglu_expert(xq, xs, *W[int(e)],
                                                                      h_quant=hq)[0]
    assert np.array_equal(out["y"][t], oracle.f64_to_bf16_bits(acc))
    # a different rounding of the same layer: close to the FP32-scale result
    W32 = {e: oracle.quantized_expert(*S.host_expert_weights(cfg, e))
           for e in range(cfg.n_routed + 1)}
    y32 = oracle.layer_forward(inp["x"], inp["router_w"], inp["bias"], cfg.n_groups,
                               cfg.topk_groups, cfg.topk, W32.__getitem__)["y"]
    a, b = S.bf16_bits_to_f32(out["y"]), S.bf16_bits_to_f32(y32)
    rel = np.linalg.norm(a - b) / np.linalg.norm(b)
    assert 0 < rel < 0.1
