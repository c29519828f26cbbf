"""Pins of the oracle's online 1x128 / 128x128 quantisation ("DeepSeek-V3
Technical Report" notes page, section "FP8 mixed precision training":
fine-grained quantisation, tile-wise 1x128 for activations and block-wise
128x128 for weights; online quantisation from the current max |value|)."""
from fractions import Fraction

import numpy as np
import torch

import oracle
import synthetic as S
from exact import e4m3_from_bits, round_to_f32


def _bf16(v):
    return S.f32_to_bf16_bits(np.asarray(v, dtype=np.float32))


def _torch_codes(v32):
    return torch.from_numpy(np.asarray(v32, np.float32)).to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_tile_with_amax_448_has_unit_scale():
    rng = np.random.default_rng(0)
    v = rng.standard_normal((3, 256)).astype(np.float32) * 40
    v[:, 17] = 448.0
    v[:, 128 + 5] = -448.0
    x = _bf16(v)
    q, s = oracle.quant_act_1x128(x)
    assert np.all(s == 1.0)
    assert np.array_equal(q, _torch_codes(S.bf16_bits_to_f32(x)))


def test_power_of_two_scale_by_hand():
    # amax = 3.5 -> scale = 3.5/448 = 2^-7 exactly, inverse 128.
    rng = np.random.default_rng(1)
    v = rng.uniform(-3.4, 3.4, size=(2, 128)).astype(np.float32)
    v[0, 3] = 3.5
    v[1, 99] = -3.5
    x = _bf16(v)
    q, s = oracle.quant_act_1x128(x)
    assert np.all(s == 2.0 ** -7)
    assert np.array_equal(q, _torch_codes(S.bf16_bits_to_f32(x) * np.float32(128)))


def test_scale_is_correctly_rounded_quotient():
    rng = np.random.default_rng(2)
    x = S.host_normal_bf16(rng, (64, 512), 1.0)
    q, s = oracle.quant_act_1x128(x)
    xf = S.bf16_bits_to_f32(x).reshape(64, 4, 128)
    amax = np.abs(xf).max(axis=2)
    for r in range(64):
        for t in range(4):
            exact = Fraction(float(amax[r, t])) / 448
            assert s[r, t] == round_to_f32(exact)
    # codes: nearest-even E4M3 of fp32(v * fp32(448/amax))
    inv = np.array([[round_to_f32(Fraction(448) / Fraction(float(a))) for a in row]
                    for row in amax], dtype=np.float32)
    prod = (xf * inv[:, :, None]).astype(np.float32).reshape(64, 512)
    assert np.array_equal(q, _torch_codes(prod))


def test_scale_invariance_under_powers_of_two():
    rng = np.random.default_rng(3)
    x = S.host_normal_bf16(rng, (8, 384), 1.0)
    q0, s0 = oracle.quant_act_1x128(x)
    for j in (-20, -3, 1, 7, 40):
        xj = _bf16(S.bf16_bits_to_f32(x) * np.float32(2.0 ** j))
        qj, sj = oracle.quant_act_1x128(xj)
        assert np.array_equal(qj, q0)
        assert np.array_equal(sj, (s0 * np.float32(2.0 ** j)).astype(np.float32))


def test_error_bound():
    rng = np.random.default_rng(4)
    x = S.host_normal_bf16(rng, (32, 1024), 1.0)
    q, s = oracle.quant_act_1x128(x)
    v = S.bf16_bits_to_f32(x).astype(np.float64)
    deq = np.array([[float(e4m3_from_bits(int(c))) for c in row] for row in q]) \
        * np.repeat(s.astype(np.float64), 128, axis=1)
    err = np.abs(deq - v)
    sc = np.repeat(s.astype(np.float64), 128, axis=1)
    normal = np.abs(v) / sc >= 2.0 ** -6
    # 3 mantissa bits: half a step is 2^-4 relative; plus the rounding of
    # v*inv to fp32 and of the scale (a few 2^-24).
    assert np.all(err[normal] <= (2.0 ** -4 + 2.0 ** -20) * np.abs(v[normal]))
    assert np.all(err[~normal] <= sc[~normal] * (2.0 ** -10 + 2.0 ** -20))


def test_zero_tile():
    x = _bf16(np.zeros((1, 256), np.float32))
    x[0, 5] = 0x8000  # -0
    q, s = oracle.quant_act_1x128(x)
    assert np.all(s == 1.0)
    assert q[0, 5] == 0x80 and np.count_nonzero(q) == 1


def test_fp32_input_path_matches_bf16_path():
    rng = np.random.default_rng(5)
    x = S.host_normal_bf16(rng, (4, 256), 1.0)
    qa, sa = oracle.quant_act_1x128(x)
    qb, sb = oracle.quant_act_1x128(S.bf16_bits_to_f32(x))
    assert np.array_equal(qa, qb) and np.array_equal(sa, sb)


def test_weight_blocks_are_independent_and_by_hand():
    rng = np.random.default_rng(6)
    w = S.host_normal_bf16(rng, (256, 384), 0.02)
    q, s = oracle.quant_w_128x128(w)
    assert s.shape == (2, 3)
    wf = S.bf16_bits_to_f32(w)
    for i in range(2):
        for j in range(3):
            blk = wf[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128]
            amax = float(np.abs(blk).max())
            assert s[i, j] == round_to_f32(Fraction(amax) / 448)
            inv = np.float32(round_to_f32(Fraction(448) / Fraction(amax)))
            assert np.array_equal(q[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128],
                                  _torch_codes((blk * inv).astype(np.float32)))
    # changing one block leaves the others untouched
    w2 = w.copy()
    w2[0:128, 0:128] = _bf16(S.bf16_bits_to_f32(w[0:128, 0:128]) * 4)
    q2, s2 = oracle.quant_w_128x128(w2)
    assert np.array_equal(q2[:, 128:], q[:, 128:]) and np.array_equal(q2[128:], q[128:])
    assert s2[0, 0] == s[0, 0] * 4 and np.array_equal(s2.ravel()[1:], s.ravel()[1:])
