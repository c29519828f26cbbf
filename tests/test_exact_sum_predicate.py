"""The no-rounding test the router's exact-sum kernel relies on, checked on
the CPU against exact rational arithmetic.

The router logit is fp32 of the FP64 sum of x_k * E_k in ascending k
("DeepSeek-V3 Technical Report" notes page, section "FP8 mixed precision
training": gating kept in high precision; the reading fixes FP64 in
ascending k).  The GPU settles an unsettled logit by a parallel sum when

    S = sum |x_k E_k|  <  2^(53 + g),   g = min over nonzero products of the
                                        exponent of the product's lowest set bit,

because every partial sum (in any order) is then a multiple of 2^g below
2^(53+g), i.e. a double, so no addition rounds.  These tests restate that
predicate in numpy and check its consequence with Fractions: wherever it
holds, the ascending-k FP64 sum and sums in other orders all equal the exact
sum; and on inputs built so that the ascending-k sum does round, the
predicate fails."""
from fractions import Fraction

import numpy as np

import synthetic as S


def _bf16_values(bits):
    return S.bf16_bits_to_f32(np.asarray(bits, dtype=np.uint16)).astype(np.float64)


def _lowbit(v: float) -> int:
    """Exponent of the lowest set bit of a nonzero double."""
    m, e = np.frexp(abs(v))          # v = m * 2^e, m in [0.5, 1)
    sig = int(m * 2.0 ** 53)         # 53-bit integer significand
    tz = (sig & -sig).bit_length() - 1
    return int(e) - 53 + tz


def _predicate(x, E) -> bool:
    p = x * E                        # bf16 x bf16: exact in FP64
    nz = p[p != 0.0]
    if nz.size == 0:
        return True
    g = min(_lowbit(float(v)) for v in nz)
    s = Fraction(0)
    for v in np.abs(nz):
        s += Fraction(float(v))      # the exact S (the GPU rounds it upward)
    return s < Fraction(2) ** (53 + g)


def _exact(x, E) -> Fraction:
    tot = Fraction(0)
    for a, b in zip(x, E):
        tot += Fraction(float(a)) * Fraction(float(b))
    return tot


def _ascending(x, E) -> float:
    acc = 0.0
    for a, b in zip(x, E):
        acc = acc + a * b
    return acc


def test_predicate_implies_order_free_exact_sum():
    rng = np.random.default_rng(17)
    held = plain_held = 0
    for trial in range(60):
        d = 256
        x = _bf16_values(S.host_normal_bf16(rng, (d,), 1.0))
        E = _bf16_values(S.host_normal_bf16(rng, (d,), 0.006))
        if trial % 3 == 1:   # values far below the row maximum
            x[rng.integers(0, d, 4)] *= 2.0 ** -30
        if trial % 3 == 2:
            E[rng.integers(0, d, 4)] *= 2.0 ** -40
        if not _predicate(x, E):
            continue
        held += 1
        plain_held += trial % 3 == 0
        ex = _exact(x, E)
        assert Fraction(_ascending(x, E)) == ex
        perm = rng.permutation(d)
        assert Fraction(_ascending(x[perm], E[perm])) == ex
        # a pairwise tree, as the warp's shuffle reduction adds
        p = list(x * E)
        while len(p) > 1:
            p = [p[i] + p[i + 1] if i + 1 < len(p) else p[i] for i in range(0, len(p), 2)]
        assert Fraction(p[0]) == ex
    # rows like the router's (no planted tiny values) pass; the planted ones
    # exercise both outcomes
    assert plain_held == 20 and held > 20


def test_predicate_fails_where_the_ascending_sum_rounds():
    # 2^40 + many 2^-40 terms: each small addition rounds away in FP64
    d = 64
    x = np.full(d, 2.0 ** -20)
    E = np.full(d, 2.0 ** -20)
    x[0], E[0] = 2.0 ** 20, 2.0 ** 20
    assert Fraction(_ascending(x, E)) != _exact(x, E)
    assert not _predicate(x, E)
    # large terms that cancel, with small ones in between
    x = np.array([2.0 ** 60, 1.0, -(2.0 ** 60), 3.0])
    E = np.array([1.0, 2.0 ** -10, 1.0, 2.0 ** -12])
    assert Fraction(_ascending(x, E)) != _exact(x, E)
    assert not _predicate(x, E)


def test_predicate_on_zero_and_single_products():
    assert _predicate(np.zeros(8), np.ones(8))
    x = np.zeros(8)
    E = np.zeros(8)
    x[3], E[3] = 3.0, -0.5
    assert _predicate(x, E)
    assert Fraction(_ascending(x, E)) == _exact(x, E)
