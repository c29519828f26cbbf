"""GPU parity of the single-GPU dispatch (expert-contiguous permutation of the
FP8 rows) and of the gate-weighted combine ("DeepSeek-V3 Technical Report"
notes page, section "DualPipe": all-to-all dispatch and combine; section
"FP8 mixed precision training": FP8 dispatch payload)."""
import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from gpu_util import DEV, need_gpu, rel_frobenius, shape_of, to_dev

pytestmark = pytest.mark.gpu


def _routing(T, N, K, rng, skew=False):
    if skew:
        p = (np.arange(1, N + 1) ** -1.5)
        p /= p.sum()
        idx = np.stack([rng.choice(N, K, replace=False, p=p) for _ in range(T)])
    else:
        idx = np.stack([rng.choice(N, K, replace=False) for _ in range(T)])
    idx = idx.astype(np.int32)
    counts = np.bincount(idx.ravel(), minlength=N).astype(np.int32)
    return idx, counts


def gpu_permute(shape, idx, counts, xq, xs):
    import fp8_block_scaled_affinity_b200 as moe
    T, K, N, d = shape.T, shape.topk, shape.n_routed, shape.d
    R = T * K + T
    xq_perm = torch.full((max(R, 1), d), 0xEE, dtype=torch.uint8, device=DEV)
    xs_perm = torch.full((d // 128, max(R, 1)), -1.0, dtype=torch.float32, device=DEV)
    off = torch.full((N + 2,), -1, dtype=torch.int32, device=DEV)
    rop = torch.full((max(T, 1), K), -1, dtype=torch.int32, device=DEV)
    ws = torch.empty((moe.moe_permute_workspace_size(shape),), dtype=torch.uint8, device=DEV)
    moe.moe_permute(shape, to_dev(idx), to_dev(counts), to_dev(xq), to_dev(xs), xq_perm, xs_perm,
                    off, rop, ws)
    torch.cuda.synchronize()
    return (xq_perm.cpu().numpy()[:R], xs_perm.cpu().numpy()[:, :R], off.cpu().numpy(),
            rop.cpu().numpy()[:T])


@pytest.mark.parametrize("T,N,K,d,skew", [(1, 16, 4, 128, False), (257, 16, 4, 512, False),
                                          (1000, 256, 8, 1024, True), (130, 64, 1, 256, False),
                                          (64, 32, 32, 128, False)])
def test_permute_bit_exact(T, N, K, d, skew):
    need_gpu()
    rng = np.random.default_rng(T + N + K)
    idx, counts = _routing(T, N, K, rng, skew)
    x = S.host_normal_bf16(rng, (T, d), 1.0)
    xq, xs = oracle.quant_act_1x128(x)   # inputs; the permutation is what is tested
    import fp8_block_scaled_affinity_b200 as moe
    shape = moe.make_shape(T, d, N, 1, 1, K, 128)
    pq, ps, off, rop = gpu_permute(shape, idx, counts, xq, xs)
    off_ref, rop_ref = oracle.permute_layout(idx, counts, N)
    assert np.array_equal(off, off_ref)
    assert np.array_equal(rop, rop_ref)
    # every routed pair and every shared row carries its token's bytes and scales
    src = np.concatenate([np.repeat(np.arange(T), K), np.arange(T)])
    rows = np.concatenate([rop_ref.ravel(), T * K + np.arange(T)])
    exp_q = np.empty_like(pq)
    exp_q[rows] = xq[src]
    exp_s = np.empty_like(ps)
    exp_s[:, rows] = xs[src].T
    assert np.array_equal(pq, exp_q)
    assert np.array_equal(ps.view(np.uint32), exp_s.view(np.uint32))


def gpu_quant_permute(shape, idx, counts, x_bits):
    import fp8_block_scaled_affinity_b200 as moe
    T, K, N, d = shape.T, shape.topk, shape.n_routed, shape.d
    R = T * K + T
    xq_perm = torch.full((max(R, 1), d), 0xEE, dtype=torch.uint8, device=DEV)
    xs_perm = torch.full((d // 128, max(R, 1)), -1.0, dtype=torch.float32, device=DEV)
    off = torch.full((N + 2,), -1, dtype=torch.int32, device=DEV)
    rop = torch.full((max(T, 1), K), -1, dtype=torch.int32, device=DEV)
    ws = torch.empty((moe.moe_permute_workspace_size(shape),), dtype=torch.uint8, device=DEV)
    x = torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).to(DEV)
    moe.moe_quant_permute(shape, x, to_dev(idx), to_dev(counts), xq_perm, xs_perm, off, rop, ws)
    torch.cuda.synchronize()
    return (xq_perm.cpu().numpy()[:R], xs_perm.cpu().numpy()[:, :R], off.cpu().numpy(),
            rop.cpu().numpy()[:T])


@pytest.mark.parametrize("T,N,K,d,skew", [(1, 16, 4, 128, False), (257, 16, 4, 512, False),
                                          (1000, 256, 8, 7168, True), (130, 64, 1, 2176, False),
                                          (64, 32, 32, 128, False)])
def test_quant_permute_bit_exact(T, N, K, d, skew):
    """The fused pass (bf16 rows quantised 1x128 straight into their K + 1
    destinations) against the oracle's quantiser and permutation: codes,
    scales, offsets and row_of_pair bit for bit.  d = 2176 (17 tiles) leaves a
    ragged last group of tiles in every row."""
    need_gpu()
    rng = np.random.default_rng(T * 7 + N + K)
    idx, counts = _routing(T, N, K, rng, skew)
    x = S.host_normal_bf16(rng, (T, d), 1.0)
    x[0, :128] = 0  # an all-zero tile: scale 1, codes 0
    xq, xs = oracle.quant_act_1x128(x)
    import fp8_block_scaled_affinity_b200 as moe
    shape = moe.make_shape(T, d, N, 1, 1, K, 128)
    pq, ps, off, rop = gpu_quant_permute(shape, idx, counts, x)
    off_ref, rop_ref = oracle.permute_layout(idx, counts, N)
    assert np.array_equal(off, off_ref)
    assert np.array_equal(rop, rop_ref)
    src = np.concatenate([np.repeat(np.arange(T), K), np.arange(T)])
    rows = np.concatenate([rop_ref.ravel(), T * K + np.arange(T)])
    exp_q = np.empty_like(pq)
    exp_q[rows] = xq[src]
    exp_s = np.empty_like(ps)
    exp_s[:, rows] = xs[src].T
    assert np.array_equal(pq, exp_q)
    assert np.array_equal(ps.view(np.uint32), exp_s.view(np.uint32))


def test_permute_empty_batch():
    import fp8_block_scaled_affinity_b200 as moe
    need_gpu()
    shape = moe.make_shape(0, 128, 16, 4, 2, 4, 128)
    _, _, off, _ = gpu_permute(shape, np.zeros((0, 4), np.int32), np.zeros(16, np.int32),
                               np.zeros((0, 128), np.uint8), np.zeros((0, 1), np.float32))
    assert off.tolist() == [0] * 18


@pytest.mark.parametrize("T,K,d", [(1, 4, 128), (300, 8, 1024), (129, 3, 7168)])
def test_combine_against_oracle(T, K, d):
    import fp8_block_scaled_affinity_b200 as moe
    need_gpu()
    rng = np.random.default_rng(T * K)
    N = 16
    idx, counts = _routing(T, N, K, rng)
    off, rop = oracle.permute_layout(idx, counts, N)
    R = T * K + T
    o = rng.standard_normal((R, d)).astype(np.float32)
    g = rng.uniform(0, 1, (T, K)).astype(np.float32)
    shape = moe.make_shape(T, d, N, 1, 1, K, 128)
    y = torch.empty((T, d), dtype=torch.bfloat16, device=DEV)
    moe.moe_combine(shape, to_dev(o), to_dev(off), to_dev(rop), to_dev(g), y)
    torch.cuda.synchronize()
    ybits = y.cpu().view(torch.int16).numpy().view(np.uint16)
    ref = oracle.combine(o[T * K:].astype(np.float64), o[rop].astype(np.float64), g)
    got = S.bf16_bits_to_f32(ybits)
    exp = S.bf16_bits_to_f32(ref)
    assert rel_frobenius(got, exp) <= 1e-3
    # fp32 accumulation may move a value across a bf16 rounding boundary, by
    # at most one bf16 step; most values agree exactly
    diff = np.abs(got.astype(np.float64) - exp)
    assert np.all(diff <= np.abs(exp) * 2.0 ** -7 + 1e-30)
    assert np.mean(ybits == ref) > 0.97


def test_update_bias_hand_example_and_equal_load():
    import fp8_block_scaled_affinity_b200 as moe
    need_gpu()
    shape = moe.make_shape(4, 128, 4, 1, 1, 2, 128, 0.125)
    counts = to_dev(np.array([3, 1, 2, 2], np.int32))
    b = to_dev(np.array([0.5, 0.25, 0.0, -0.125], np.float32))
    moe.moe_update_bias(shape, counts, b)
    torch.cuda.synchronize()
    assert b.cpu().numpy().tolist() == [0.375, 0.375, 0.0, -0.125]
