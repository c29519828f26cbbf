"""Pins of the oracle's routing ("DeepSeek-V3 Technical Report" notes page,
section "DeepSeekMoE and auxiliary-loss-free load balancing": sigmoid
affinity, a per-expert bias added for the routing decision only, gates from
the normalised selected (unbiased) affinities, tokens sent to at most M nodes,
per-batch load monitoring and the gamma update, no token dropping)."""
import itertools
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synthetic as S
from conftest import read_golden
from exact import bf16_bits_to_fraction, round_to_f32, sigmoid_f32


def _golden():
    rows = {}
    for r in read_golden("route_hand.txt"):
        rows.setdefault(r[0], []).append([float(v) for v in r[1:]])
    return rows


def _hand_inputs():
    g = _golden()
    u = np.array(g["u"][0], np.float32)
    d = 128
    x = np.zeros((2, d), np.float32)
    x[0, 0], x[1, 0] = 1.0, -1.0
    E = np.zeros((8, d), np.float32)
    E[:, 0] = u
    return g, S.f32_to_bf16_bits(x), S.f32_to_bf16_bits(E), np.array(g["bias"][0], np.float32)


def test_hand_worked_example():
    g, x, E, b = _hand_inputs()
    r = oracle.route(x, E, b, n_groups=4, topk_groups=2, topk=3, want_scores=True)
    assert r["topk_idx"].tolist() == [[int(v) for v in row] for row in g["topk_idx"]]
    assert r["counts"].tolist() == [int(v) for v in g["counts"][0]]
    # gates: selected unbiased sigmoid values, normalised (decimal sigmoid)
    for t, sgn in ((0, 1.0), (1, -1.0)):
        sel = r["topk_idx"][t]
        s = [sigmoid_f32(sgn * float(g["u"][0][i])) for i in sel]
        tot = sum(Fraction(v) for v in s)
        exp = [round_to_f32(Fraction(v) / tot) for v in s]
        assert r["topk_gate"][t].tolist() == exp
    new_b = oracle.update_bias(r["counts"], b, T=2, topk=3, gamma=0.001)
    sign = np.array(g["bias_sign"][0])
    assert np.array_equal(new_b, (b + np.float32(0.001) * sign.astype(np.float32)).astype(np.float32))
    off, rop = oracle.permute_layout(r["topk_idx"], r["counts"], 8)
    assert off.tolist() == [int(v) for v in g["offsets"][0]]
    assert rop.tolist() == [[int(v) for v in row] for row in g["row_of_pair"]]


def _exact_logit(xrow, erow) -> float:
    """fp32 rounding of the exact sum of bf16 products (integer arithmetic)."""
    tot = Fraction(0)
    for a, b in zip(xrow.tolist(), erow.tolist()):
        if a & 0x7FFF and b & 0x7FFF:
            tot += bf16_bits_to_fraction(a) * bf16_bits_to_fraction(b)
    return round_to_f32(tot)


def test_logits_equal_correctly_rounded_exact_sums():
    cfg = S.CONFIGS["tiny"]
    inp = S.make_layer_inputs_host(cfg)
    x, E = inp["x"][:12], inp["router_w"]
    r = oracle.route(x, E, inp["bias"], cfg.n_groups, cfg.topk_groups, cfg.topk,
                     want_scores=True)
    for t in range(12):
        for i in range(cfg.n_routed):
            assert r["logits"][t, i] == _exact_logit(x[t], E[i]), (t, i)


def test_sigmoid_against_high_precision_decimal():
    cfg = S.CONFIGS["tiny"]
    inp = S.make_layer_inputs_host(cfg)
    r = oracle.route(inp["x"][:40], inp["router_w"], inp["bias"], cfg.n_groups,
                     cfg.topk_groups, cfg.topk, want_scores=True)
    u, s = r["logits"], r["scores"]
    for t in range(40):
        for i in range(cfg.n_routed):
            assert s[t, i] == sigmoid_f32(float(u[t, i]))
    # wide range of logits, including saturating ones
    for uu in (-30.0, -8.5, -1e-3, 0.0, 1e-7, 3.25, 17.0, 40.0):
        x = np.zeros((1, 128), np.float32)
        x[0, 0] = 1.0
        E = np.zeros((4, 128), np.float32)
        E[:, 0] = uu
        rr = oracle.route(S.f32_to_bf16_bits(x), S.f32_to_bf16_bits(E),
                          np.zeros(4, np.float32), 1, 1, 2, want_scores=True)
        ub = float(rr["logits"][0, 0])
        assert rr["scores"][0, 0] == sigmoid_f32(ub)


def _brute_force(sb, n_groups, M, K):
    """Best M-subset of groups by sum of group maxima, then best K-subset of the
    candidate experts by sum of biased scores (exhaustive enumeration)."""
    n = len(sb)
    ng = n // n_groups
    gmax = [max(sb[g * ng:(g + 1) * ng]) for g in range(n_groups)]
    best_g = max(itertools.combinations(range(n_groups), M),
                 key=lambda c: sum(Fraction(float(gmax[g])) for g in c))
    cand = [i for i in range(n) if i // ng in best_g]
    best_e = max(itertools.combinations(cand, K),
                 key=lambda c: sum(Fraction(float(sb[i])) for i in c))
    return set(best_g), set(best_e)


@pytest.mark.parametrize("n_routed,n_groups,M,K,seed", [
    (16, 4, 2, 4, 0), (12, 3, 2, 3, 1), (16, 8, 3, 4, 2), (8, 2, 1, 2, 3),
    (16, 1, 1, 5, 4), (10, 5, 5, 6, 5)])
def test_selection_matches_brute_force(n_routed, n_groups, M, K, seed):
    rng = np.random.default_rng(seed)
    T, d = 24, 256
    x = S.host_normal_bf16(rng, (T, d), 1.0)
    E = S.host_normal_bf16(rng, (n_routed, d), 0.05)
    b = S.host_uniform_f32(rng, (n_routed,), 0.1)
    r = oracle.route(x, E, b, n_groups, M, K, want_scores=True)
    s = r["scores"]
    sb = (s + b[None, :]).astype(np.float32)   # one IEEE fp32 add per entry
    ng = n_routed // n_groups
    for t in range(T):
        gsel, esel = _brute_force(sb[t], n_groups, M, K)
        got = r["topk_idx"][t].tolist()
        assert set(got) == esel
        assert len({i // ng for i in got}) <= M
        assert {i // ng for i in got} <= gsel
        # slots in descending biased score
        vals = [sb[t, i] for i in got]
        assert vals == sorted(vals, reverse=True)


def test_gates_normalised_and_from_unbiased_scores():
    cfg = S.CONFIGS["tiny"]
    inp = S.make_layer_inputs_host(cfg)
    r = oracle.route(inp["x"], inp["router_w"], inp["bias"], cfg.n_groups,
                     cfg.topk_groups, cfg.topk, want_scores=True)
    g = r["topk_gate"].astype(np.float64)
    assert np.all(np.abs(g.sum(1) - 1.0) <= cfg.topk * 2.0 ** -24)
    s = r["scores"]
    for t in range(0, cfg.T, 7):
        sel = r["topk_idx"][t]
        tot = sum(Fraction(float(s[t, i])) for i in sel)
        assert r["topk_gate"][t].tolist() == [round_to_f32(Fraction(float(s[t, i])) / tot)
                                             for i in sel]


def test_bias_only_affects_selection():
    cfg = S.CONFIGS["tiny"]
    inp = S.make_layer_inputs_host(cfg)
    args = (cfg.n_groups, cfg.topk_groups, cfg.topk)
    r0 = oracle.route(inp["x"], inp["router_w"], np.zeros(cfg.n_routed, np.float32), *args)
    r1 = oracle.route(inp["x"], inp["router_w"], inp["bias"], *args)
    same = np.all(np.sort(r0["topk_idx"], 1) == np.sort(r1["topk_idx"], 1), axis=1)
    assert same.sum() > 10 and (~same).sum() > 0
    for t in np.nonzero(same)[0]:
        g0 = dict(zip(r0["topk_idx"][t].tolist(), r0["topk_gate"][t].tolist()))
        g1 = dict(zip(r1["topk_idx"][t].tolist(), r1["topk_gate"][t].tolist()))
        assert g0 == g1


def test_raising_a_bias_attracts_and_keeps_tokens():
    cfg = S.CONFIGS["tiny"]
    inp = S.make_layer_inputs_host(cfg)
    args = (cfg.n_groups, cfg.topk_groups, cfg.topk)
    r = oracle.route(inp["x"], inp["router_w"], inp["bias"], *args)
    b = inp["bias"].copy()
    b[5] += np.float32(0.003)
    r2 = oracle.route(inp["x"], inp["router_w"], b, *args)
    had = np.any(r["topk_idx"] == 5, axis=1)
    has = np.any(r2["topk_idx"] == 5, axis=1)
    assert np.all(has[had])               # selected tokens stay selected
    assert r2["counts"][5] >= r["counts"][5]
    b[5] += np.float32(5.0)               # dominates every token's choice
    r3 = oracle.route(inp["x"], inp["router_w"], b, *args)
    assert r3["counts"][5] == cfg.T


def test_counts_are_the_histogram_and_nothing_is_dropped():
    cfg = S.CONFIGS["tiny"]
    inp = S.make_layer_inputs_host(cfg)
    r = oracle.route(inp["x"], inp["router_w"], inp["bias"], cfg.n_groups,
                     cfg.topk_groups, cfg.topk)
    assert r["counts"].sum() == cfg.T * cfg.topk
    assert np.array_equal(r["counts"], np.bincount(r["topk_idx"].ravel(), minlength=cfg.n_routed))
    for row in r["topk_idx"]:
        assert len(set(row.tolist())) == cfg.topk


def test_logit_offset_is_added_to_the_logit():
    cfg = S.CONFIGS["tiny"]
    inp = S.make_layer_inputs_host(cfg)
    off = S.zipf_logit_offset(cfg.n_routed, 1.2)
    r0 = oracle.route(inp["x"][:8], inp["router_w"], inp["bias"], cfg.n_groups,
                      cfg.topk_groups, cfg.topk, want_scores=True)
    r1 = oracle.route(inp["x"][:8], inp["router_w"], inp["bias"], cfg.n_groups,
                      cfg.topk_groups, cfg.topk, logit_offset=off, want_scores=True)
    assert np.array_equal(r1["logits"], (r0["logits"] + off[None, :]).astype(np.float32))


def test_route_rejects_bad_group_shape():
    x = np.zeros((1, 128), np.uint16)
    E = np.zeros((10, 128), np.uint16)
    with pytest.raises(ValueError):
        oracle.route(x, E, np.zeros(10, np.float32), 3, 1, 2)
    with pytest.raises(ValueError):
        oracle.route(x, E, np.zeros(10, np.float32), 5, 1, 3)  # 1 group of 2 < K


def test_ties_go_to_the_lower_index():
    """Reading (pages silent on ties): equal group scores and equal biased
    affinities resolve to the lower group / expert index.  All 8 experts get
    the same logit, so groups 0 and 1 and experts 0, 1, 2 win (by hand)."""
    x = np.zeros((2, 128), np.float32)
    x[:, 0] = 1.0
    E = np.zeros((8, 128), np.float32)
    E[:, 0] = 0.75
    b = np.zeros(8, np.float32)
    r = oracle.route(S.f32_to_bf16_bits(x), S.f32_to_bf16_bits(E), b, 4, 2, 3)
    assert r["topk_idx"].tolist() == [[0, 1, 2], [0, 1, 2]]
    # a tie only inside the later group: experts 5 and 4 equal, above the rest
    E[4, 0] = E[5, 0] = 2.0
    r = oracle.route(S.f32_to_bf16_bits(x), S.f32_to_bf16_bits(E), b, 4, 2, 3)
    assert r["topk_idx"].tolist() == [[4, 5, 0], [4, 5, 0]]
