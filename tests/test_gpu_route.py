"""GPU parity of routing, load histogram and bias update against the oracle,
bit for bit ("DeepSeek-V3 Technical Report" notes page, section "DeepSeekMoE
and auxiliary-loss-free load balancing")."""
import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from conftest import read_golden
from gpu_util import DEV, bf16_dev, need_gpu, shape_of, to_dev

pytestmark = pytest.mark.gpu


def gpu_route(shape, xbits, Ebits, bias, offset=None):
    import fp8_block_scaled_affinity_b200 as moe
    T, K, N = shape.T, shape.topk, shape.n_routed
    idx = torch.full((max(T, 1), K), -1, dtype=torch.int32, device=DEV)
    gate = torch.full((max(T, 1), K), -1.0, dtype=torch.float32, device=DEV)
    counts = torch.full((N,), 77, dtype=torch.int32, device=DEV)
    ws = torch.empty((max(moe.moe_route_workspace_size(shape), 1),), dtype=torch.uint8, device=DEV)
    moe.moe_route(shape, bf16_dev(xbits) if T else None, bf16_dev(Ebits), to_dev(bias),
                  None if offset is None else to_dev(offset), idx, gate, counts, ws)
    torch.cuda.synchronize()
    return idx.cpu().numpy()[:T], gate.cpu().numpy()[:T], counts.cpu().numpy()


def _compare(cfg, inp, T=None, offset=None):
    T = cfg.T if T is None else T
    shape = shape_of(cfg, T)
    x = inp["x"][:T]
    idx, gate, counts = gpu_route(shape, x, inp["router_w"], inp["bias"], offset)
    ref = oracle.route(x, inp["router_w"], inp["bias"], cfg.n_groups, cfg.topk_groups,
                       cfg.topk, logit_offset=offset)
    assert np.array_equal(idx, ref["topk_idx"])
    assert np.array_equal(gate.view(np.uint32), ref["topk_gate"].view(np.uint32))
    assert np.array_equal(counts, ref["counts"])
    return ref


def test_hand_worked_example():
    need_gpu()
    g = {}
    for r in read_golden("route_hand.txt"):
        g.setdefault(r[0], []).append([float(v) for v in r[1:]])
    x = np.zeros((2, 128), np.float32)
    x[0, 0], x[1, 0] = 1.0, -1.0
    E = np.zeros((8, 128), np.float32)
    E[:, 0] = g["u"][0]
    import fp8_block_scaled_affinity_b200 as moe
    shape = moe.make_shape(2, 128, 8, 4, 2, 3, 128, 0.001)
    idx, gate, counts = gpu_route(shape, S.f32_to_bf16_bits(x), S.f32_to_bf16_bits(E),
                                  np.array(g["bias"][0], np.float32))
    assert idx.tolist() == [[int(v) for v in row] for row in g["topk_idx"]]
    assert counts.tolist() == [int(v) for v in g["counts"][0]]


def test_ties_go_to_lower_index():
    import fp8_block_scaled_affinity_b200 as moe
    need_gpu()
    x = np.zeros((3, 128), np.float32)
    x[:, 0] = 1.0
    E = np.zeros((8, 128), np.float32)
    E[:, 0] = 0.75
    shape = moe.make_shape(3, 128, 8, 4, 2, 3, 128)
    idx, _, _ = gpu_route(shape, S.f32_to_bf16_bits(x), S.f32_to_bf16_bits(E),
                          np.zeros(8, np.float32))
    assert idx.tolist() == [[0, 1, 2]] * 3


def _compare_arrays(x, E, bias, G, M, K, offset=None):
    import fp8_block_scaled_affinity_b200 as moe
    T, d = x.shape
    N = E.shape[0]
    shape = moe.make_shape(T, d, N, G, M, K, 128)
    idx, gate, counts = gpu_route(shape, x, E, bias, offset)
    ref = oracle.route(x, E, bias, G, M, K, logit_offset=offset)
    assert np.array_equal(idx, ref["topk_idx"])
    assert np.array_equal(gate.view(np.uint32), ref["topk_gate"].view(np.uint32))
    assert np.array_equal(counts, ref["counts"])
    return ref


@pytest.mark.parametrize("T", [200, 700])
def test_fully_tied_router(T):
    """A zero router: every logit is 0 and every biased score ties, so no
    token's choice can be decided from bounds; every token gets all of its
    logits from the defining FP64 sums (one sum per thread for a short list,
    FP64 tiles for a long one) and the ties go to the lower indices."""
    need_gpu()
    rng = np.random.default_rng(T)
    x = S.host_normal_bf16(rng, (T, 256), 1.0)
    E = np.zeros((64, 256), np.uint16)
    ref = _compare_arrays(x, E, np.zeros(64, np.float32), 8, 2, 6)
    assert (ref["topk_idx"] == np.arange(6)).all()


def test_duplicated_router_rows():
    """Pairs of identical router rows with equal biases tie exactly; tokens
    whose K-th and (K+1)-th choices are such a pair need the exact path,
    the others are decided from bounds."""
    need_gpu()
    rng = np.random.default_rng(11)
    T, d, N = 512, 384, 64
    x = S.host_normal_bf16(rng, (T, d), 1.0)
    E = S.host_normal_bf16(rng, (N, d), 0.05)
    E[1::2] = E[0::2]
    bias = S.host_uniform_f32(rng, (N,), 0.02)
    bias[1::2] = bias[0::2]
    _compare_arrays(x, E, bias, 4, 2, 5)


def test_huge_cancelling_entries():
    """Entries near 1e30 times router entries near 3e8: the products reach
    the top of the fp32 range (their fp32 bound is useless, so the tokens go
    to the exact path) and cancel exactly in the FP64 sum, which must widen
    both factors to FP64 before multiplying."""
    need_gpu()
    rng = np.random.default_rng(5)
    T, d, N = 64, 256, 32
    xf = rng.standard_normal((T, d)).astype(np.float32)
    xf[:, 0], xf[:, 1] = 1e30, -1e30
    Ef = (rng.standard_normal((N, d)) * 0.05).astype(np.float32)
    c = rng.uniform(1.7e8, 3.0e8, N).astype(np.float32)
    Ef[:, 0] = c
    Ef[:, 1] = c
    x, E = S.f32_to_bf16_bits(xf), S.f32_to_bf16_bits(Ef)
    _compare_arrays(x, E, S.host_uniform_f32(rng, (N,), 0.02), 4, 2, 4)


@pytest.mark.parametrize("T", [1, 37, 256])
def test_tiny_workload(T):
    need_gpu()
    cfg = S.CONFIGS["tiny"]
    _compare(cfg, S.make_layer_inputs_host(cfg), T=T)


@pytest.mark.parametrize("n_routed,n_groups,M,K", [(64, 8, 3, 6), (96, 32, 7, 12),
                                                   (1024, 16, 4, 32), (48, 1, 1, 5)])
def test_other_routing_shapes(n_routed, n_groups, M, K):
    need_gpu()
    rng = np.random.default_rng(n_routed + K)
    T, d = 150, 384
    inp = {"x": S.host_normal_bf16(rng, (T, d), 1.0),
           "router_w": S.host_normal_bf16(rng, (n_routed, d), 0.05),
           "bias": S.host_uniform_f32(rng, (n_routed,), 0.02)}
    cfg = S.MoeConfig("t", T, d, n_routed, n_groups, M, K, 128, 0.05, 0.02, 0.001, 0)
    _compare(cfg, inp)


def test_decode_workload_full():
    need_gpu()
    cfg = S.CONFIGS["decode"]
    _compare(cfg, S.make_layer_inputs_host(cfg))


def test_prefill_workload_full():
    need_gpu()
    cfg = S.CONFIGS["prefill"]
    _compare(cfg, S.make_layer_inputs_host(cfg))


def test_skewed_workload_eight_batches_with_bias_updates():
    """Eight successive batches of 16384 tokens with a Zipf(1.2) logit prior;
    after each batch the bias moves by gamma.  Routing, counts and the bias
    trajectory must match the oracle's own trajectory bit for bit."""
    import fp8_block_scaled_affinity_b200 as moe
    need_gpu()
    cfg = S.CONFIGS["skewed"]
    shape = shape_of(cfg)
    base = S.make_layer_inputs_host(cfg, 0)
    off = base["logit_offset"]
    b_gpu = to_dev(base["bias"])
    b_ref = base["bias"].copy()
    E = base["router_w"]
    loads = []
    for j in range(cfg.batches):
        x = S.make_layer_inputs_host(cfg, j)["x"]
        idx = torch.empty((cfg.T, cfg.topk), dtype=torch.int32, device=DEV)
        gate = torch.empty((cfg.T, cfg.topk), dtype=torch.float32, device=DEV)
        counts = torch.empty((cfg.n_routed,), dtype=torch.int32, device=DEV)
        ws = torch.empty((moe.moe_route_workspace_size(shape),), dtype=torch.uint8, device=DEV)
        moe.moe_route(shape, bf16_dev(x), bf16_dev(E), b_gpu, to_dev(off), idx, gate, counts, ws)
        moe.moe_update_bias(shape, counts, b_gpu)
        torch.cuda.synchronize()
        ref = oracle.route(x, E, b_ref, cfg.n_groups, cfg.topk_groups, cfg.topk, logit_offset=off)
        assert np.array_equal(idx.cpu().numpy(), ref["topk_idx"]), j
        assert np.array_equal(gate.cpu().numpy().view(np.uint32),
                              ref["topk_gate"].view(np.uint32)), j
        assert np.array_equal(counts.cpu().numpy(), ref["counts"]), j
        b_ref = oracle.update_bias(ref["counts"], b_ref, cfg.T, cfg.topk, cfg.gamma)
        assert np.array_equal(b_gpu.cpu().numpy().view(np.uint32), b_ref.view(np.uint32)), j
        c = ref["counts"]
        loads.append(c.max() / c.mean())
    assert loads[0] > 3.0  # the prior really skews the load


def test_empty_batch_zeroes_counts():
    import fp8_block_scaled_affinity_b200 as moe
    need_gpu()
    cfg = S.CONFIGS["tiny"]
    inp = S.make_layer_inputs_host(cfg)
    shape = shape_of(cfg, 0)
    _, _, counts = gpu_route(shape, inp["x"][:0], inp["router_w"], inp["bias"])
    assert np.all(counts == 0)
    bad = moe.make_shape(4, 128, 10, 3, 1, 2, 128)  # N_r % G != 0
    with pytest.raises(moe.MoeError):
        gpu_route(bad, inp["x"][:4, :128], inp["router_w"][:10, :128], inp["bias"][:10])


# ----------------------------------------------------------------------
# Near ties: biased scores a few fp32 ulps apart without being equal.
#
# The router certifies each token's choice from intervals around scores
# computed from exact integer logits; an interval that is too narrow would
# certify a wrong choice exactly when two candidates are one or two ulps
# apart.  Here every router row is the same base row except in its own
# "perturbation slot", an element whose value is tiny (2^-e for a spread of
# e), so all N_r logits of a token agree except in their last few bits:
# every group boundary and every K-th / (K+1)-th boundary is a near tie.

def _near_tie_router(N, d, rng):
    base = S.bf16_bits_to_f32(S.host_normal_bf16(rng, (d,), 0.02)).astype(np.float32)
    slots = np.arange(N) * (d // N)  # one slot per expert, spread over k
    base[slots] = 0.0
    E = np.tile(base, (N, 1))
    # slot value 2^-e with e from 14 to 24: the logit differences x_k 2^-e
    # then span a few ulps of |u| ~ 1
    e = 14 + (np.arange(N) * 7) % 11
    E[np.arange(N), slots] = np.ldexp(1.0, -e).astype(np.float32)
    return S.f32_to_bf16_bits(E)


@pytest.mark.parametrize("N,G,M,K,d", [(16, 4, 2, 4, 512), (64, 8, 4, 8, 1024),
                                       (256, 8, 4, 8, 7168)])
def test_near_tied_scores_bit_exact(N, G, M, K, d):
    import fp8_block_scaled_affinity_b200 as moe
    need_gpu()
    rng = np.random.default_rng(N + d)
    T = 1024
    E = _near_tie_router(N, d, rng)
    x = S.host_normal_bf16(rng, (T, d), 1.0)
    bias = np.zeros(N, np.float32)  # equal biases keep the scores' last bits in play
    shape = moe.make_shape(T, d, N, G, M, K, 256, 0.001)
    idx, gate, counts = gpu_route(shape, x, E, bias)
    ref = oracle.route(x, E, bias, G, M, K, want_scores=True)
    assert np.array_equal(idx, ref["topk_idx"])
    assert np.array_equal(gate.view(np.uint32), ref["topk_gate"].view(np.uint32))
    assert np.array_equal(counts, ref["counts"])
    # the case is adversarial: count tokens whose K-th and (K+1)-th best
    # biased scores (over all experts) are 1 or 2 fp32 ulps apart
    s = np.sort(ref["scores"].astype(np.float32) + bias, axis=1)[:, ::-1]
    gap = s[:, K - 1].view(np.int32).astype(np.int64) - s[:, K].view(np.int32).astype(np.int64)
    assert np.sum((gap >= 1) & (gap <= 2)) >= T // 20


@pytest.mark.parametrize("T", [3, 200])
def test_near_tied_short_list(T):
    """Few tokens, all near ties: the uncertified list stays short, so every
    logit of a listed token is summed by one thread in ascending k (fp32
    products where the rows allow, FP64 otherwise), at the full width."""
    import fp8_block_scaled_affinity_b200 as moe
    need_gpu()
    N, G, M, K, d = 256, 8, 4, 8, 7168
    rng = np.random.default_rng(T + 17)
    E = _near_tie_router(N, d, rng)
    x = S.host_normal_bf16(rng, (T, d), 1.0)
    bias = np.zeros(N, np.float32)
    shape = moe.make_shape(T, d, N, G, M, K, 256, 0.001)
    idx, gate, counts = gpu_route(shape, x, E, bias)
    ref = oracle.route(x, E, bias, G, M, K)
    assert np.array_equal(idx, ref["topk_idx"])
    assert np.array_equal(gate.view(np.uint32), ref["topk_gate"].view(np.uint32))
    assert np.array_equal(counts, ref["counts"])


def test_near_tied_scores_with_offsets_and_biases():
    """The same near-tied router with a logit offset and biases that differ
    by single ulps."""
    import fp8_block_scaled_affinity_b200 as moe
    need_gpu()
    N, G, M, K, d, T = 64, 8, 4, 8, 1024, 1024
    rng = np.random.default_rng(5)
    E = _near_tie_router(N, d, rng)
    x = S.host_normal_bf16(rng, (T, d), 1.0)
    b0 = np.float32(0.0125)
    step = np.arange(N, dtype=np.int32)
    bias = (np.full(N, b0, np.float32).view(np.int32) + step % 3).view(np.float32)
    offset = (np.full(N, -1.5, np.float32).view(np.int32) + step % 2).view(np.float32)
    assert bias.shape == (N,) and offset.shape == (N,) and np.isfinite(offset).all()
    shape = moe.make_shape(T, d, N, G, M, K, 256, 0.001)
    idx, gate, counts = gpu_route(shape, x, E, bias, offset)
    ref = oracle.route(x, E, bias, G, M, K, logit_offset=offset)
    assert np.array_equal(idx, ref["topk_idx"])
    assert np.array_equal(gate.view(np.uint32), ref["topk_gate"].view(np.uint32))
    assert np.array_equal(counts, ref["counts"])


def test_pageable_host_pointer_is_rejected_not_dereferenced():
    """A pageable host array passed where device memory is expected (here the
    logit offset) returns MOE_ERR_ARG before any kernel is launched."""
    import fp8_block_scaled_affinity_b200 as moe
    need_gpu()
    cfg = S.CONFIGS["tiny"]
    inp = S.make_layer_inputs_host(cfg, 0)
    shape = shape_of(cfg, 64)
    idx = torch.empty((64, cfg.topk), dtype=torch.int32, device=DEV)
    gate = torch.empty((64, cfg.topk), dtype=torch.float32, device=DEV)
    counts = torch.empty((cfg.n_routed,), dtype=torch.int32, device=DEV)
    ws = torch.empty((moe.moe_route_workspace_size(shape),), dtype=torch.uint8, device=DEV)
    host_offset = torch.zeros(cfg.n_routed, dtype=torch.float32)  # pageable host memory
    with pytest.raises(moe.MoeError) as e:
        moe.moe_route(shape, bf16_dev(inp["x"][:64]), bf16_dev(inp["router_w"]),
                      to_dev(inp["bias"]), host_offset, idx, gate, counts, ws)
    assert e.value.status == -7
    torch.cuda.synchronize()


@pytest.mark.parametrize("cfg_name,T,with_offset", [("tiny", 256, False), ("skewed", 2048, True)])
def test_route_scores_are_the_chosen_unbiased_affinities(cfg_name, T, with_offset):
    """moe_route_scores writes, besides moe_route's outputs (bit-identical),
    the unbiased affinity s of each chosen expert in slot order, equal to
    the oracle's s at those experts bit for bit (the values the gates are
    normalised from and the backward pass differentiates)."""
    need_gpu()
    import fp8_block_scaled_affinity_b200 as moe
    cfg = S.CONFIGS[cfg_name]
    inp = S.make_layer_inputs_host(cfg, 0)
    x = inp["x"][:T]
    off = inp["logit_offset"] if with_offset else None
    shape = shape_of(cfg, T)
    K, N = cfg.topk, cfg.n_routed
    idx = torch.empty((T, K), dtype=torch.int32, device=DEV)
    gate = torch.empty((T, K), dtype=torch.float32, device=DEV)
    score = torch.empty((T, K), dtype=torch.float32, device=DEV)
    counts = torch.empty((N,), dtype=torch.int32, device=DEV)
    ws = torch.empty((moe.moe_route_workspace_size(shape),), dtype=torch.uint8, device=DEV)
    moe.moe_route_scores(shape, bf16_dev(x), bf16_dev(inp["router_w"]), to_dev(inp["bias"]),
                         None if off is None else to_dev(off), idx, gate, score, counts, ws)
    torch.cuda.synchronize()
    ref = oracle.route(x, inp["router_w"], inp["bias"], cfg.n_groups, cfg.topk_groups, K,
                       logit_offset=off, want_scores=True)
    assert np.array_equal(idx.cpu().numpy(), ref["topk_idx"])
    assert np.array_equal(gate.cpu().numpy().view(np.uint32), ref["topk_gate"].view(np.uint32))
    assert np.array_equal(counts.cpu().numpy(), ref["counts"])
    s_ref = np.take_along_axis(ref["scores"], ref["topk_idx"], axis=1)
    assert np.array_equal(score.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
