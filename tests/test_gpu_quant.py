"""GPU parity of the online FP8 quantisers against the oracle, bit for bit
("DeepSeek-V3 Technical Report" notes page, section "FP8 mixed precision
training": 1x128 activation tiles, 128x128 weight blocks, E4M3, online
max-abs scaling)."""
import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from gpu_util import DEV, bf16_dev, need_gpu

pytestmark = pytest.mark.gpu


def _gpu_act(xbits, kb_major=False):
    import fp8_block_scaled_affinity_b200 as moe
    x = bf16_dev(xbits)
    rows, cols = xbits.shape
    q = torch.empty((rows, cols), dtype=torch.uint8, device=DEV)
    s = torch.empty((cols // 128, rows) if kb_major else (rows, cols // 128),
                    dtype=torch.float32, device=DEV)
    moe.fp8_quant_act_1x128(x, q, s, kb_major)
    torch.cuda.synchronize()
    s = s.cpu().numpy()
    return q.cpu().numpy(), (s.T.copy() if kb_major else s)


def test_every_bf16_value_with_unit_scale():
    """All 65536 bf16 patterns (NaN/inf excluded) through tiles whose amax is
    448, so the scale is 1 and the code is the plain E4M3 cast."""
    need_gpu()
    allv = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    f = S.bf16_bits_to_f32(allv)
    keep = allv[np.isfinite(f) & (np.abs(f) <= 448.0)]
    per = 127
    n_tiles = (keep.size + per - 1) // per
    tiles = np.zeros((n_tiles, 128), dtype=np.uint16)
    flat = np.concatenate([keep, np.zeros(n_tiles * per - keep.size, np.uint16)])
    tiles[:, :per] = flat.reshape(n_tiles, per)
    tiles[:, per] = S.f32_to_bf16_bits(np.array([448.0], np.float32))[0]
    x = tiles.reshape(-1, 512) if n_tiles % 4 == 0 else tiles
    q, s = _gpu_act(x)
    qo, so = oracle.quant_act_1x128(x)
    assert np.array_equal(s, so) and np.all(s == 1.0)
    assert np.array_equal(q, qo)


@pytest.mark.parametrize("rows,cols,kb_major", [(1, 128, False), (7, 384, False),
                                                (333, 1024, True), (4097, 256, True),
                                                (3, 7168, False)])
def test_random_activations_bit_exact(rows, cols, kb_major):
    need_gpu()
    rng = np.random.default_rng(rows * 31 + cols)
    v = rng.standard_normal((rows, cols)).astype(np.float32)
    v *= np.where(rng.random((rows, cols)) < 0.001, 100.0, 1.0).astype(np.float32)
    v[0, :128] = 0.0                      # an all-zero tile
    if rows > 2:
        v[2, 5] = -0.0
        v[1, :128] *= np.float32(2.0 ** -30)   # tiny values: subnormal codes
    x = S.f32_to_bf16_bits(v)
    q, s = _gpu_act(x, kb_major)
    qo, so = oracle.quant_act_1x128(x)
    assert np.array_equal(s, so)
    assert np.array_equal(q, qo)


def test_full_size_prefill_activations_bit_exact():
    need_gpu()
    cfg = S.CONFIGS["prefill"]
    x = S.make_layer_inputs_host(cfg)["x"]
    q, s = _gpu_act(x, kb_major=False)
    qo, so = oracle.quant_act_1x128(x)
    assert np.array_equal(s, so) and np.array_equal(q, qo)


@pytest.mark.parametrize("rows,cols", [(128, 128), (256, 384), (640, 1152)])
def test_weight_blocks_bit_exact(rows, cols):
    import fp8_block_scaled_affinity_b200 as moe
    need_gpu()
    rng = np.random.default_rng(rows + cols)
    v = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    v[:128, :128] = 0.0
    if cols > 128:
        v[:128, 128:256] *= np.float32(1e4)
    w = S.f32_to_bf16_bits(v)
    q = torch.empty((rows, cols), dtype=torch.uint8, device=DEV)
    s = torch.empty((rows // 128, cols // 128), dtype=torch.float32, device=DEV)
    moe.fp8_quant_w_128x128(bf16_dev(w), q, s)
    torch.cuda.synchronize()
    qo, so = oracle.quant_w_128x128(w)
    assert np.array_equal(s.cpu().numpy(), so)
    assert np.array_equal(q.cpu().numpy(), qo)


def test_full_size_expert_weights_bit_exact():
    """One full-size expert (W1, W3, W2 of the prefill workload)."""
    import fp8_block_scaled_affinity_b200 as moe
    from gpu_util import expert_bf16, host_bits
    need_gpu()
    cfg = S.CONFIGS["prefill"]
    for w in expert_bf16(cfg, 7):
        rows, cols = w.shape
        q = torch.empty((rows, cols), dtype=torch.uint8, device=DEV)
        s = torch.empty((rows // 128, cols // 128), dtype=torch.float32, device=DEV)
        moe.fp8_quant_w_128x128(w, q, s)
        torch.cuda.synchronize()
        qo, so = oracle.quant_w_128x128(host_bits(w))
        assert np.array_equal(s.cpu().numpy(), so)
        assert np.array_equal(q.cpu().numpy(), qo)


def test_host_side_rejections():
    import fp8_block_scaled_affinity_b200 as moe
    need_gpu()
    x = torch.zeros((4, 100), dtype=torch.bfloat16, device=DEV)
    q = torch.empty((4, 100), dtype=torch.uint8, device=DEV)
    s = torch.empty((4, 1), dtype=torch.float32, device=DEV)
    with pytest.raises(moe.MoeError) as e:
        moe.fp8_quant_act_1x128(x, q, s)
    assert e.value.status == -2
    x = torch.zeros((0, 128), dtype=torch.bfloat16, device=DEV)
    moe.fp8_quant_act_1x128(x, q, s)  # empty input: nothing to do
