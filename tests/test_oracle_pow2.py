"""Pins of the oracle's power-of-two scale option (a numerically different
option, not the pages' FP32-scale recipe): scale = 2^e with e the smallest
integer such that amax <= 448 * 2^e, codes = E4M3(v * 2^-e).  The E4M3
encoding itself is pinned in test_oracle_e4m3.py; here the exponent rule is
checked with exact rationals, the codes against torch's float8_e4m3fn cast
of the exactly scaled values, and the invariances the rule implies."""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synthetic as S


def _e_ref(amax):
    """Smallest integer e with amax <= 448 * 2^e, by exact search."""
    if amax == 0:
        return 0
    a = Fraction(float(amax))
    e = 0
    while a > 448 * Fraction(2) ** e:
        e += 1
    while a <= 448 * Fraction(2) ** (e - 1):
        e -= 1
    return e


@pytest.mark.parametrize("amax,e", [(448.0, 0), (449.0, 1), (896.0, 1), (897.0, 2),
                                    (1.0, -8), (0.875, -9), (0.8750001, -8), (224.0, -1),
                                    (224.00002, 0), (2.0 ** -20, -28)])
def test_hand_exponents(amax, e):
    row = np.zeros((1, 128), np.float32)
    row[0, 5] = -amax
    row[0, 9] = amax / 3
    q, ee = oracle.quant_act_1x128_pow2(row)
    assert ee[0, 0] == e == _e_ref(np.float32(amax))
    # the largest magnitude maps to at most 448 and more than 224
    v = abs(np.float64(np.float32(amax))) * 2.0 ** -e
    assert 224 < v <= 448


def test_exponent_is_minimal_and_codes_match_torch():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((64, 1024)).astype(np.float32)
    x *= np.ldexp(1.0, rng.integers(-30, 30, (64, 1))).astype(np.float32)
    xb = S.f32_to_bf16_bits(x)
    xf = S.bf16_bits_to_f32(xb)
    q, e = oracle.quant_act_1x128_pow2(xb)
    amax = np.abs(xf.reshape(64, 8, 128)).max(axis=2)
    for r in range(64):
        for t in range(8):
            assert e[r, t] == _e_ref(amax[r, t])
    scaled = (xf.reshape(64, 8, 128) * np.ldexp(1.0, -e)[:, :, None].astype(np.float32)).reshape(64, 1024)
    ref = torch.from_numpy(scaled).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, ref)


def test_power_of_two_invariance_and_zero_tiles():
    rng = np.random.default_rng(4)
    x = S.bf16_bits_to_f32(S.f32_to_bf16_bits(rng.standard_normal((8, 256)).astype(np.float32)))
    q0, e0 = oracle.quant_act_1x128_pow2(x)
    for j in (-7, 3, 20):
        q1, e1 = oracle.quant_act_1x128_pow2((x * np.float32(2.0 ** j)).astype(np.float32))
        assert np.array_equal(q0, q1) and np.array_equal(e1, e0 + j)
    z = np.zeros((2, 128), np.float32)
    z[1] = -0.0
    q, e = oracle.quant_act_1x128_pow2(z)
    assert np.all(e == 0) and np.all(q[0] == 0x00) and np.all(q[1] == 0x80)


def test_weight_blocks_pow2():
    rng = np.random.default_rng(5)
    w = S.host_normal_bf16(rng, (256, 384), 0.006)
    wf = S.bf16_bits_to_f32(w)
    q, e = oracle.quant_w_128x128_pow2(w)
    assert e.shape == (2, 3)
    for i in range(2):
        for j in range(3):
            blk = wf[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128]
            assert e[i, j] == _e_ref(np.abs(blk).max())
            scaled = blk * np.float32(2.0 ** -int(e[i, j]))
            ref = torch.from_numpy(np.ascontiguousarray(scaled)).to(
                torch.float8_e4m3fn).view(torch.uint8).numpy()
            assert np.array_equal(q[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128], ref)
    # dequantised within the E4M3 error bound of the original
    deq = oracle.e4m3_decode_table()[q] * np.repeat(np.repeat(oracle.pow2_scales(e), 128, 0), 128, 1)
    rel = np.abs(deq - wf) / np.maximum(np.abs(wf), 1e-30)
    normal = np.abs(wf) >= np.repeat(np.repeat(oracle.pow2_scales(e), 128, 0), 128, 1) * 2.0 ** -6
    assert rel[normal].max() <= 2.0 ** -4
