"""Exact rational helpers for pinning the oracle (tests only).

Independent of ``oracle/``: values are decoded from bit patterns by the
IEEE/OCP definitions and rounded with integer arithmetic, so a mistake in
the oracle's FP64 route does not repeat here.
"""
from __future__ import annotations

from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np


def bf16_bits_to_fraction(b: int) -> Fraction:
    b = int(b) & 0xFFFF
    s = -1 if b >> 15 else 1
    e = (b >> 7) & 0xFF
    m = b & 0x7F
    if e == 0:
        return s * Fraction(m, 1 << 7) * Fraction(1, 1 << 126)
    assert e != 0xFF
    return s * Fraction(128 + m, 128) * (Fraction(2) ** (e - 127))


def f32_to_fraction(x: float) -> Fraction:
    return Fraction(float(np.float32(x)))


def _round_fraction(v: Fraction, mant_bits: int, emin: int, emax_val: Fraction):
    """Round rational v to the binary grid with ``mant_bits`` significant bits
    (including the leading one), minimum normal exponent emin; nearest, ties
    to even.  Returns a Fraction (may exceed emax_val: caller saturates)."""
    if v == 0:
        return Fraction(0)
    sign = -1 if v < 0 else 1
    a = abs(v)
    # exponent e with 2^e <= a < 2^(e+1)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    if Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, emin)
    step = Fraction(2) ** (e - (mant_bits - 1))
    q = a / step
    n = q.numerator // q.denominator
    rem = q - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return sign * n * step


def round_to_f32(v: Fraction) -> float:
    r = _round_fraction(v, 24, -126, None)
    return float(np.float32(float(r)))  # exact: r is an fp32 value


def round_to_bf16_bits(v: Fraction) -> int:
    r = _round_fraction(v, 8, -126, None)
    f = np.float32(float(r))
    return int(np.array([f], dtype=np.float32).view(np.uint32)[0] >> 16)


def e4m3_from_bits(c: int):
    """OCP E4M3 value of a code as a Fraction (None for NaN)."""
    s = -1 if c & 0x80 else 1
    e = (c >> 3) & 15
    m = c & 7
    if e == 15 and m == 7:
        return None
    if e == 0:
        return s * Fraction(m, 512)
    return s * Fraction(8 + m, 8) * Fraction(2) ** (e - 7)


def sigmoid_f32(u: float, digits: int = 50) -> float:
    """fp32(1 / (1 + exp(-u))) with exp evaluated in decimal at ``digits``."""
    getcontext().prec = digits
    du = Decimal(float(u))
    s = Decimal(1) / (Decimal(1) + (-du).exp())
    return round_to_f32(Fraction(s))


def silu_fraction(a: Fraction, digits: int = 50) -> Fraction:
    getcontext().prec = digits
    da = Decimal(a.numerator) / Decimal(a.denominator)
    return Fraction(da / (Decimal(1) + (-da).exp()))
