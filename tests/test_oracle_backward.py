"""Pins of the oracle's backward (gate, router and expert-MLP gradients)
against central finite differences of the forward definitions in FP64, with
the FP8 quantisation points switched off (the quantisers are pinned on their
own) and the top-K selection held fixed (it is piecewise constant)."""
import numpy as np
import pytest

import oracle
import synthetic as S


def _num_grad(f, x, h=1e-6):
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        xp, xm = x.copy(), x.copy()
        xp[i] += h
        xm[i] -= h
        g[i] = (f(xp) - f(xm)) / (2 * h)
    return g


def test_gate_backward_matches_finite_differences():
    rng = np.random.default_rng(0)
    T, K, d = 3, 4, 8
    u = rng.standard_normal((T, K))
    o = rng.standard_normal((T, K, d))
    dy_f = rng.standard_normal((T, d)).astype(np.float32)
    dy = S.f32_to_bf16_bits(dy_f)
    dyv = S.bf16_bits_to_f32(dy).astype(np.float64)

    def loss(uu):
        s = 1.0 / (1.0 + np.exp(-uu))
        g = s / s.sum(axis=1, keepdims=True)
        return float(np.einsum("td,tk,tkd->", dyv, g, o))
    s = 1.0 / (1.0 + np.exp(-u))
    dg, du = oracle.gate_backward(dy, o, s.astype(np.float32))
    # the oracle rounds s to fp32 as the forward stores it: compare at 1e-6
    num = _num_grad(loss, u)
    assert np.allclose(du, num, rtol=1e-5, atol=1e-6)
    assert np.allclose(dg, np.einsum("td,tkd->tk", dyv, o))


def test_router_backward_matches_finite_differences():
    rng = np.random.default_rng(1)
    T, K, N, d = 4, 2, 5, 6
    x = S.f32_to_bf16_bits(rng.standard_normal((T, d)).astype(np.float32))
    E = S.f32_to_bf16_bits(rng.standard_normal((N, d)).astype(np.float32))
    idx = np.array([[0, 3], [1, 4], [3, 2], [0, 1]], np.int32)
    du = rng.standard_normal((T, K))
    xv, Ev = S.bf16_bits_to_f32(x).astype(np.float64), S.bf16_bits_to_f32(E).astype(np.float64)
    dx, dE = oracle.router_backward(du, idx, x, E)

    def loss_x(xx):
        return float(sum(du[t, k] * xx[t] @ Ev[idx[t, k]] for t in range(T) for k in range(K)))

    def loss_E(EE):
        return float(sum(du[t, k] * xv[t] @ EE[idx[t, k]] for t in range(T) for k in range(K)))
    assert np.allclose(dx, _num_grad(loss_x, xv), atol=1e-7)
    assert np.allclose(dE, _num_grad(loss_E, Ev), atol=1e-7)


def test_expert_backward_matches_finite_differences():
    """Unquantised chain: y(x) = (silu(x W1^T) * (x W3^T)) W2^T, L = <do, y>."""
    rng = np.random.default_rng(2)
    rows, d, I = 3, 128, 128
    w = [oracle.quant_w_128x128(S.host_normal_bf16(rng, sh, 0.05))
         for sh in ((I, d), (I, d), (d, I))]
    W1, W3, W2 = (oracle.dequant_w(*m) for m in w)
    x = rng.standard_normal((rows, d))
    do = rng.standard_normal((rows, d)).astype(np.float32)

    def loss(xx):
        a, c = xx @ W1.T, xx @ W3.T
        y = (a / (1.0 + np.exp(-a)) * c) @ W2.T
        return float(np.sum(do.astype(np.float64) * y))
    got = oracle.expert_backward(do, x, None, *w, quant=False)
    num = _num_grad(loss, x, h=1e-5)
    assert np.allclose(got, num, rtol=1e-5, atol=1e-6)
    # with the FP8 quantisation points: the same gradient within FP8 error
    xq, xs = oracle.quant_act_1x128(x.astype(np.float32))
    q = oracle.expert_backward(do, xq, xs, *w)
    rel = np.linalg.norm(q - num) / np.linalg.norm(num)
    assert rel < 0.1


def test_swiglu_backward_matches_finite_differences():
    rng = np.random.default_rng(3)
    a, c, dh = (rng.standard_normal((4, 6)) * 3 for _ in range(3))

    def h(aa, cc):
        return aa / (1.0 + np.exp(-aa)) * cc
    da, dc = oracle.swiglu_backward(dh, a, c)
    eps = 1e-6
    assert np.allclose(da, dh * (h(a + eps, c) - h(a - eps, c)) / (2 * eps), rtol=1e-6,
                       atol=1e-8)
    assert np.allclose(dc, dh * (h(a, c + eps) - h(a, c - eps)) / (2 * eps), rtol=1e-6,
                       atol=1e-8)


def test_layer_backward_matches_finite_differences():
    """The whole layer's dx (shared expert, gated routed experts, router
    through the gates) against central differences of the unquantised FP64
    forward with the top-K choice held at the one the oracle's router makes;
    and dE likewise.  A dropped shared-expert term, a wrong gate or a missing
    router term each moves dx far outside the tolerance."""
    rng = np.random.default_rng(4)
    T, d, N, G, M, K, I = 3, 128, 4, 2, 2, 2, 128
    x = S.f32_to_bf16_bits(rng.standard_normal((T, d)).astype(np.float32))
    E = S.f32_to_bf16_bits((rng.standard_normal((N, d)) * 0.1).astype(np.float32))
    bias = (rng.standard_normal(N) * 0.01).astype(np.float32)
    dy = S.f32_to_bf16_bits(rng.standard_normal((T, d)).astype(np.float32))
    ws = [oracle.quantized_expert(*(S.host_normal_bf16(rng, sh, 0.1)
                                    for sh in ((I, d), (I, d), (d, I))))
          for _ in range(N + 1)]
    got = oracle.layer_backward(dy, x, E, bias, G, M, K, lambda e: ws[e], quant=False)
    idx = got["topk_idx"]
    W = [[oracle.dequant_w(*m) for m in w] for w in ws]
    dyv = S.bf16_bits_to_f32(dy).astype(np.float64)

    def expert(e, X):
        W1, W3, W2 = W[e]
        a, c = X @ W1.T, X @ W3.T
        return (a / (1.0 + np.exp(-a)) * c) @ W2.T

    def loss(X, Ev):
        s = 1.0 / (1.0 + np.exp(-(X @ Ev.T)))
        sk = np.take_along_axis(s, idx, axis=1)
        g = sk / sk.sum(axis=1, keepdims=True)
        y = expert(N, X)
        for t in range(T):
            for k in range(K):
                y[t] += g[t, k] * expert(idx[t, k], X[t:t + 1])[0]
        return float(np.sum(dyv * y))
    xv = S.bf16_bits_to_f32(x).astype(np.float64)
    Ev = S.bf16_bits_to_f32(E).astype(np.float64)
    num_dx = _num_grad(lambda X: loss(X, Ev), xv, h=1e-5)
    num_dE = _num_grad(lambda EE: loss(xv, EE), Ev, h=1e-5)
    scale_x, scale_E = np.abs(num_dx).max(), np.abs(num_dE).max()
    assert np.abs(got["dx"] - num_dx).max() <= 1e-5 * scale_x
    assert np.abs(got["dE"] - num_dE).max() <= 1e-5 * scale_E


def test_quant_act_128x1_blocks_follow_the_rows():
    """Blocks of 128 rows from the first row, one scale per column and
    block, stored transposed; the ragged last block is padded with zero
    codes.  Every (block, column) gets a distinct amax, so a transposed or
    shifted index moves a scale to the wrong place."""
    rows, cols = 300, 5
    rng = np.random.default_rng(5)
    x = rng.uniform(-1.0, 1.0, (rows, cols)).astype(np.float32)
    amax = np.zeros((3, cols), np.float32)
    for b in range(3):
        for j in range(cols):
            a = np.float32(2.0 + 3 * b + 0.25 * j)
            r = 128 * b + (7 * j + 3 * b) % min(128, rows - 128 * b)
            x[r, j] = -a if (b + j) % 2 else a
            amax[b, j] = a
    q, s = oracle.quant_act_128x1(x)
    assert q.shape == (cols, 384) and s.shape == (cols, 3)
    assert np.allclose(s.T * 448.0, amax, rtol=1e-6)
    assert np.all(q[:, rows:] == 0)
    deq = oracle.dequant_act(q, s)[:, :rows].T
    assert np.all(np.abs(deq - x) <= 2.0**-4 * np.abs(x) + 2.0**-9 * np.repeat(s.T, 128, 0)[:rows])


def test_layer_weight_gradients_match_finite_differences():
    """dW1, dW3, dW2 of every expert (shared one included) from the
    unquantised chain against central differences of the FP64 forward in a
    sample of weight entries; an expert no token chose has zero gradients."""
    rng = np.random.default_rng(6)
    T, d, N, G, M, K, I = 3, 128, 4, 2, 2, 2, 128
    x = S.f32_to_bf16_bits(rng.standard_normal((T, d)).astype(np.float32))
    E = S.f32_to_bf16_bits((rng.standard_normal((N, d)) * 0.1).astype(np.float32))
    bias = np.array([0.0, 0.0, 0.0, -5.0], np.float32)  # expert 3 is never chosen
    dy = S.f32_to_bf16_bits(rng.standard_normal((T, d)).astype(np.float32))
    ws = [oracle.quantized_expert(*(S.host_normal_bf16(rng, sh, 0.1)
                                    for sh in ((I, d), (I, d), (d, I))))
          for _ in range(N + 1)]
    got = oracle.layer_backward(dy, x, E, bias, G, M, K, lambda e: ws[e], quant=False,
                                wgrad_experts=tuple(range(N + 1)))
    idx = got["topk_idx"]
    assert not np.any(idx == 3)
    W = [[oracle.dequant_w(*m) for m in w] for w in ws]
    xv = S.bf16_bits_to_f32(x).astype(np.float64)
    Ev = S.bf16_bits_to_f32(E).astype(np.float64)
    dyv = S.bf16_bits_to_f32(dy).astype(np.float64)
    s = 1.0 / (1.0 + np.exp(-(xv @ Ev.T)))
    sk = np.take_along_axis(s, idx, axis=1)
    g = sk / sk.sum(axis=1, keepdims=True)

    def loss(Wl):
        def expert(e, X):
            W1, W3, W2 = Wl[e]
            a, c = X @ W1.T, X @ W3.T
            return (a / (1.0 + np.exp(-a)) * c) @ W2.T
        y = expert(N, xv)
        for t in range(T):
            for k in range(K):
                y[t] += g[t, k] * expert(idx[t, k], xv[t:t + 1])[0]
        return float(np.sum(dyv * y))
    h = 1e-5
    for e in range(N + 1):
        dW13, dW2 = got["dW"][e]
        grads = (dW13[:I], dW13[I:], dW2)
        for m in range(3):
            for _ in range(12):
                i, j = rng.integers(0, W[e][m].shape[0]), rng.integers(0, W[e][m].shape[1])
                Wp = [[w.copy() for w in we] for we in W]
                Wm = [[w.copy() for w in we] for we in W]
                Wp[e][m][i, j] += h
                Wm[e][m][i, j] -= h
                num = (loss(Wp) - loss(Wm)) / (2 * h)
                scale = max(np.abs(grads[m]).max(), 1e-12)
                assert abs(grads[m][i, j] - num) <= 1e-6 * scale + 1e-9, (e, m, i, j)
        if e == 3:
            assert not np.any(dW13) and not np.any(dW2)


def test_gemm_wgrad_brute_force():
    """The K-grouped GEMM against a loop over groups, rows, columns and K
    with each product scaled by its row's and column's block scales; an
    empty group is zero."""
    rng = np.random.default_rng(7)
    m, n, nkb = 3, 2, 4
    table = oracle.e4m3_decode_table()
    finite = np.nonzero(np.isfinite(table))[0].astype(np.uint8)
    a = rng.choice(finite, (m, 128 * nkb))
    b = rng.choice(finite, (n, 128 * nkb))
    sa = rng.uniform(0.5, 2.0, (nkb, m)).astype(np.float32)
    sb = rng.uniform(0.5, 2.0, (nkb, n)).astype(np.float32)
    kb_off = np.array([0, 1, 1, 4], np.int32)
    got = oracle.gemm_wgrad(a, sa, b, sb, kb_off)
    for g in range(3):
        for i in range(m):
            for j in range(n):
                ref = 0.0
                for k in range(128 * kb_off[g], 128 * kb_off[g + 1]):
                    kb = k // 128
                    ref += float(table[a[i, k]]) * float(sa[kb, i]) * float(table[b[j, k]]) * \
                        float(sb[kb, j])
                assert abs(got[g, i, j] - ref) <= 1e-9 * max(1.0, abs(ref))
    assert not np.any(got[1])
