"""CPU pin of the router's certification bound.

The GPU router computes every logit from exact integer products of the rows'
truncated 28-bit integer parts (four 7-bit digit planes on the tensor cores)
and decides a token's routing from intervals around the resulting scores.
This file restates, from the mathematics, the bound it relies on and checks
that the bound really covers the distance it claims to cover, with exact
rational arithmetic, on random rows and on rows built to be hard:

  u~ = fl64(2^(sx + se - 56) * sum_k X_k Y_k)   (X, Y: rows truncated to
       multiples of 2^(s - 28), s the exponent of the row's largest value)
  |u~ - u_def| <= B = r1(x) max|E| + r1(E) max|x| + g_d ||x||_2 ||E||_2
                      + 2^-52 |u~| + 1e-300
  where u_def is the defining FP64 sum of x_k E_k in ascending k, r1 the
  sum of the truncated remainders, g_d = d u / (1 - d u) (1 + 2^-20) with
  u = 2^-53, and the row norms and remainder sums raised by
  1 + 4 (d + 64) 2^-53 + 2^-50 to cover their own FP64 evaluation.

and that the interval [c - delta, c + delta] of the biased score, with
  c = 1 / (1 + exp(-(u~ + off))) + b,  B' = B + 2^-23 (|u~| + |off| + B),
  delta = B' / 4 + 2^-23 + 2^-24 |b| + 1e-14,
holds the defining biased score s' = fp32(fp32(sigmoid(fp32(fp32(u_def) +
off))) + b) ("DeepSeek-V3 Technical Report" notes page, section
"DeepSeekMoE and auxiliary-loss-free load balancing": sigmoid affinity plus
the bias; gating kept in high precision per section "FP8 mixed precision
training")."""
import math
from fractions import Fraction

import numpy as np
import pytest

import synthetic as S

U = 2.0 ** -53


def _slice(v):
    """Integer parts and statistics of one row (float64 values of bf16)."""
    mx = float(np.max(np.abs(v)))
    sigma = math.frexp(mx)[1] if mx > 0 else 0  # mx < 2^sigma
    unit = math.ldexp(1.0, sigma - 28)
    X = np.trunc(v / unit)                       # exact: |v / unit| < 2^28
    rem = v - X * unit                           # exact
    return X.astype(np.int64), unit, float(np.sum(np.abs(rem))), mx


def _bound_pieces(x, e):
    d = x.size
    nmargin = 4.0 * (d + 64) * U + 2.0 ** -50
    gamma = (d * U / (1.0 - d * U)) * (1.0 + 2.0 ** -20)
    X, ux, r1x, mxx = _slice(x)
    Y, ue, r1e, mxe = _slice(e)
    exact_int = int(np.dot(X.astype(object), Y.astype(object)))  # Python ints: exact
    u_t = float(Fraction(exact_int) * Fraction(ux) * Fraction(ue))  # one rounding
    l2x = math.sqrt(float(np.sum(x * x))) * (1 + nmargin)
    l2e = math.sqrt(float(np.sum(e * e))) * (1 + nmargin)
    r1x *= 1 + nmargin
    r1e *= 1 + nmargin
    B = r1x * mxe + r1e * mxx + gamma * l2x * l2e + 2.0 ** -52 * abs(u_t) + 1e-300
    return u_t, B


def _u_def(x, e):
    s = 0.0
    for a, b in zip(x.tolist(), e.tolist()):
        s += a * b  # each product of two bf16 values is exact in FP64
    return s


def _bf16(v):
    return S.bf16_bits_to_f32(S.f32_to_bf16_bits(np.asarray(v, np.float32))).astype(np.float64)


def _rows(kind, d, rng):
    if kind == "normal":
        return _bf16(rng.standard_normal(d)), _bf16(rng.standard_normal(d) * 0.006)
    if kind == "wide_range":
        # values spread over 2^-40 .. 2^10: many remainders below the unit
        ex = rng.integers(-40, 10, d)
        return (_bf16(np.ldexp(rng.standard_normal(d), ex)),
                _bf16(np.ldexp(rng.standard_normal(d), rng.integers(-30, 0, d))))
    if kind == "wide_range_e":
        # the router row carries the remainders, the token row slices exactly
        ex = rng.integers(-36, 0, d)
        return _bf16(rng.standard_normal(d)), _bf16(np.ldexp(rng.standard_normal(d), ex))
    if kind == "exact_slices_rounding_sum":
        # both rows slice exactly (every value within 2^21 of the row's
        # maximum) but the FP64 running sum rounds at almost every step
        big = rng.random(d) < 0.5
        x = _bf16(np.where(big, 2.0 ** 20, 1.0) * rng.choice([-1.0, 1.0], d) * (1 + rng.random(d)))
        e = _bf16(np.where(big, 2.0 ** 20, 1.0) * (1 + rng.random(d)))
        return x, e
    if kind == "cancelling":
        # large values that cancel pairwise, and small ones that survive
        a = _bf16(rng.standard_normal(d // 2) * 1e4)
        x = np.empty(d)
        x[0::2], x[1::2] = a, -a
        x[::7] = _bf16(rng.standard_normal(x[::7].size) * 1e-3)
        return x, _bf16(np.abs(rng.standard_normal(d)) + 1.0)
    if kind == "rounding_heavy":
        # a running sum that rounds at nearly every step in FP64
        x = _bf16(np.where(np.arange(d) % 2 == 0, 2.0 ** 40, 1.0 + rng.random(d)))
        e = _bf16(np.where(np.arange(d) % 2 == 0, 1.0, rng.random(d) * 2.0 ** -3))
        x[0] = _bf16(np.array([3.0 ** 20]))[0]
        return x, e
    if kind == "tiny":
        # near the bottom of the bf16 range (products far below 2^-126)
        return (_bf16(np.ldexp(rng.standard_normal(d), -120)),
                _bf16(np.ldexp(rng.standard_normal(d), -20)))
    raise ValueError(kind)


@pytest.mark.parametrize("kind", ["normal", "wide_range", "wide_range_e", "cancelling",
                                  "rounding_heavy", "exact_slices_rounding_sum", "tiny"])
@pytest.mark.parametrize("d", [128, 1024, 7168])
def test_logit_bound_covers_the_defining_sum(kind, d):
    rng = np.random.default_rng(d + len(kind))
    for _ in range(3):
        x, e = _rows(kind, d, rng)
        u_t, B = _bound_pieces(x, e)
        dist = abs(Fraction(u_t) - Fraction(_u_def(x, e)))
        assert dist <= Fraction(B), (kind, d, float(dist), B)


def test_logit_bound_is_not_vacuous_on_typical_rows():
    """On ordinary rows the bound is far below a logit's fp32 ulp, so it
    settles almost every choice (else the certification would be useless)."""
    rng = np.random.default_rng(0)
    x, e = _rows("normal", 7168, rng)
    u_t, B = _bound_pieces(x, e)
    assert B < 2.0 ** -30 * max(abs(u_t), 1.0)


def _sigmoid64(u):
    """1 / (1 + exp(-u)) in FP64 (exp overflows to +inf for very negative u)."""
    with np.errstate(over="ignore"):
        return float(1.0 / (1.0 + np.exp(-np.float64(u))))


def _score_def(u_def, off, b):
    u = np.float32(u_def)
    u = np.float32(np.float64(u) + np.float64(off)) if off is not None else u
    s = np.float32(_sigmoid64(u))
    return np.float32(np.float64(s) + np.float64(b))


@pytest.mark.parametrize("kind", ["normal", "wide_range", "wide_range_e", "cancelling",
                                  "rounding_heavy", "exact_slices_rounding_sum"])
def test_score_interval_holds_the_defining_biased_score(kind):
    rng = np.random.default_rng(17 + len(kind))
    for trial in range(40):
        x, e = _rows(kind, 1024, rng)
        u_t, B = _bound_pieces(x, e)
        u_def = _u_def(x, e)
        off = None if trial % 2 else float(np.float32(rng.uniform(-7, 0)))
        b = float(np.float32(rng.uniform(-0.05, 0.05)))
        offv = 0.0 if off is None else off
        Bp = B + 2.0 ** -23 * (abs(u_t) + abs(offv) + B)
        c = _sigmoid64(u_t + offv) + b
        delta = 0.25 * Bp + 2.0 ** -23 + 2.0 ** -24 * abs(b) + 1e-14
        lo = np.nextafter(np.float32(c - delta), np.float32(-np.inf))  # rounded outwards
        hi = np.nextafter(np.float32(c + delta), np.float32(np.inf))
        s = _score_def(u_def, off, b)
        assert lo <= s <= hi, (kind, trial, float(lo), float(s), float(hi))
