"""Pins of the oracle's E4M3 codec ("DeepSeek-V3 Technical Report" notes page,
section "FP8 mixed precision training": E4M3 for every tensor; format details
from the OCP FP8 standard)."""
import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden
from exact import e4m3_from_bits


def test_decode_matches_hand_table():
    table = oracle.e4m3_decode_table()
    for code_s, val_s in read_golden("e4m3_codes.txt"):
        c = int(code_s, 16)
        if val_s == "nan":
            assert np.isnan(table[c])
        else:
            v = float(val_s)
            assert table[c] == v, (hex(c), table[c], v)
            if val_s == "-0":
                assert np.signbit(table[c])


def test_decode_matches_bit_definition_and_torch():
    table = oracle.e4m3_decode_table()
    codes = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn)
    via_torch = codes.to(torch.float64).numpy()
    for c in range(256):
        ref = e4m3_from_bits(c)
        if ref is None:
            assert np.isnan(table[c]) and np.isnan(via_torch[c])
        else:
            assert table[c] == float(ref) == via_torch[c]


def test_round_trip_all_codes():
    table = oracle.e4m3_decode_table()
    finite = [c for c in range(256) if not np.isnan(table[c])]
    vals = np.array([table[c] for c in finite], dtype=np.float32)
    enc = oracle.e4m3_encode(vals)
    assert list(enc) == finite  # both zeros keep their sign


def _torch_encode(v: np.ndarray) -> np.ndarray:
    return torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


@pytest.mark.parametrize("exp_lo,exp_hi", [(-12, -4), (-1, 1), (6, 8)])
def test_encode_exhaustive_mantissas_vs_torch(exp_lo, exp_hi):
    """Every fp32 mantissa for the given exponents, both signs, against torch's
    nearest-even cast (a library routine).  torch does not saturate (it maps
    >= 464 to NaN), so values at or above 464 are checked separately."""
    mant = np.arange(1 << 23, dtype=np.uint32)
    for e in range(exp_lo, exp_hi + 1):
        bits = ((np.uint32(e + 127) << np.uint32(23)) | mant)
        v = bits.view(np.float32)
        v = v[np.abs(v) < 464.0]
        for sgn in (1.0, -1.0):
            x = (v * np.float32(sgn)).astype(np.float32)
            assert np.array_equal(oracle.e4m3_encode(x), _torch_encode(x)), e


def test_encode_random_and_subnormal_fp32_vs_torch():
    rng = np.random.default_rng(123)
    bits = rng.integers(0, 1 << 32, size=4_000_000, dtype=np.uint64).astype(np.uint32)
    v = bits.view(np.float32)
    v = v[np.isfinite(v) & (np.abs(v) < 464.0)]
    assert np.array_equal(oracle.e4m3_encode(v), _torch_encode(v))
    tiny = np.arange(0, 1 << 23, 97, dtype=np.uint32).view(np.float32)  # fp32 subnormals
    assert np.all(oracle.e4m3_encode(tiny) == 0)


def test_encode_saturates():
    v = np.array([448.0, 463.99, 464.0, 480.0, 1e6, 3.4e38, np.inf,
                  -464.0, -1e6, -np.inf], dtype=np.float32)
    assert list(oracle.e4m3_encode(v)) == [0x7E] * 7 + [0xFE] * 3


def test_encode_ties_to_even():
    # 1 + 1/16 lies halfway between 1 (mantissa 0) and 1.125 (mantissa 1)
    # -> even -> 1.0; 1 + 3/16 halfway between 1.125 and 1.25 -> 1.25.
    # Subnormal: 0.5 * 2^-9 -> 0; 1.5 * 2^-9 -> 2 * 2^-9.
    v = np.array([1.0625, 1.1875, 2.0 ** -10, 1.5 * 2.0 ** -9, 2.5 * 2.0 ** -9],
                 dtype=np.float32)
    assert list(oracle.e4m3_encode(v)) == [0x38, 0x3A, 0x00, 0x02, 0x02]
