"""GPU parity of the power-of-two scale option (UE8M0 scale bytes and the
block-scaled tensor-core GEMM) against the oracle's power-of-two mode.

This is a numerically different option beside the pages' FP32-scale recipe
("DeepSeek-V3 Technical Report" notes page, section "FP8 mixed precision
training", and its discussion of hardware support for tile / block
quantisation): scale bytes and codes are bit-exact; GEMM outputs are
compared element by element against FP64 over the dequantised operands with
the bound of FP32 accumulation over the whole K range (the scales are exact
powers of two, applied inside the MMA)."""
import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from gpu_util import DEV, bf16_dev, need_gpu, rel_frobenius, to_dev

pytestmark = pytest.mark.gpu


def _q_act(xbits, kb_major=True):
    import fp8_block_scaled_affinity_b200 as moe
    rows, cols = xbits.shape
    q = torch.empty((rows, cols), dtype=torch.uint8, device=DEV)
    sf = torch.empty((cols // 128, rows) if kb_major else (rows, cols // 128), dtype=torch.uint8,
                     device=DEV)
    moe.fp8_quant_act_1x128_ue8m0(bf16_dev(xbits), q, sf, kb_major)
    return q, sf


def _q_w(wbits):
    import fp8_block_scaled_affinity_b200 as moe
    rows, cols = wbits.shape
    q = torch.empty((rows, cols), dtype=torch.uint8, device=DEV)
    sf = torch.empty((rows // 128, cols // 128), dtype=torch.uint8, device=DEV)
    moe.fp8_quant_w_128x128_ue8m0(bf16_dev(wbits), q, sf)
    return q, sf


@pytest.mark.parametrize("kb_major", [False, True])
def test_activation_quantiser_bit_exact(kb_major):
    need_gpu()
    rng = np.random.default_rng(11)
    x = rng.standard_normal((515, 1024)).astype(np.float32)
    x *= np.ldexp(1.0, rng.integers(-40, 40, (515, 8))).repeat(128, axis=1).astype(np.float32)
    x[3] = 0.0
    xb = S.f32_to_bf16_bits(x)
    q, sf = _q_act(xb, kb_major)
    qo, eo = oracle.quant_act_1x128_pow2(xb)
    assert np.array_equal(q.cpu().numpy(), qo)
    got = sf.cpu().numpy()
    got = got.T if kb_major else got
    assert np.array_equal(got.astype(np.int32) - 127, eo)


def test_weight_quantiser_bit_exact():
    need_gpu()
    rng = np.random.default_rng(12)
    w = S.host_normal_bf16(rng, (512, 768), 0.006)
    q, sf = _q_w(w)
    qo, eo = oracle.quant_w_128x128_pow2(w)
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(sf.cpu().numpy().astype(np.int32) - 127, eo)


def _run_mx(sizes, k, n, epilogue, seed, pad_rows=3):
    import fp8_block_scaled_affinity_b200 as moe
    rng = np.random.default_rng(seed)
    G = len(sizes)
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    R = int(off[-1]) + pad_rows
    a = S.f32_to_bf16_bits(rng.standard_normal((R, k)).astype(np.float32))
    w = S.host_normal_bf16(rng, (G * n, k), 0.05)
    aq, asf = _q_act(a, True)
    wq, wsf = _q_w(w)
    if epilogue == moe.MOE_EPI_SWIGLU_QUANT:
        out = torch.full((R, n // 2), 0xEE, dtype=torch.uint8, device=DEV)
        out_sf = torch.full((n // 256, R), 0xEE, dtype=torch.uint8, device=DEV)
    elif epilogue == moe.MOE_EPI_F32:
        out = torch.full((R, n), float("nan"), dtype=torch.float32, device=DEV)
        out_sf = None
    else:
        out = torch.full((R, n), float("nan"), dtype=torch.bfloat16, device=DEV)
        out_sf = None
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    moe.moe_grouped_gemm_mxfp8(G, to_dev(off), R, aq, asf, k, wq, wsf, n, epilogue, out, out_sf,
                               status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    qa, ea = oracle.quant_act_1x128_pow2(a)
    table = oracle.e4m3_decode_table()
    X = table[qa] * np.repeat(oracle.pow2_scales(ea), 128, axis=1)
    res = []
    for g in range(G):
        r0, r1 = off[g], off[g + 1]
        qw, ew = oracle.quant_w_128x128_pow2(w[g * n:(g + 1) * n])
        W = table[qw] * np.repeat(np.repeat(oracle.pow2_scales(ew), 128, 0), 128, 1)
        res.append((X[r0:r1], W))
    return out, out_sf, res, off


def _rank(codes):
    c = codes.astype(np.int32)
    return np.where(c & 0x80, -(c & 0x7F), c & 0x7F)


@pytest.mark.parametrize("sizes,k,n", [([1], 128, 256), ([300, 0, 17, 129], 512, 512),
                                       ([16, 32, 64, 65, 200], 384, 768)])
def test_mx_gemm_fp32_element_wise(sizes, k, n):
    import fp8_block_scaled_affinity_b200 as moe
    need_gpu()
    out, _, res, off = _run_mx(sizes, k, n, moe.MOE_EPI_F32, seed=sum(sizes) + n)
    got = out.cpu().numpy().astype(np.float64)
    for g, (X, W) in enumerate(res):
        r0, r1 = off[g], off[g + 1]
        if r1 == r0:
            continue
        ref = X @ W.T
        # FP32 accumulation of exact products over the whole K range
        bound = 2.0 ** -23 * (k + 2) * (np.abs(X) @ np.abs(W).T)
        err = np.abs(got[r0:r1] - ref)
        assert not (err > bound).any(), (g, float(err.max()))
        assert rel_frobenius(got[r0:r1], ref) <= 1e-5
    assert np.all(np.isnan(got[off[-1]:]))


def test_mx_gemm_many_items_bf16():
    """64 groups of 130-300 rows: every CTA runs several items (the
    accumulator hand-over between items); bf16 out."""
    import fp8_block_scaled_affinity_b200 as moe
    need_gpu()
    sizes = np.random.default_rng(77).integers(130, 301, size=64).tolist()
    out, _, res, off = _run_mx(sizes, 512, 1024, moe.MOE_EPI_BF16, seed=78)
    got = S.bf16_bits_to_f32(out.cpu().view(torch.int16).numpy().view(np.uint16))
    for g, (X, W) in enumerate(res):
        r0, r1 = off[g], off[g + 1]
        ref = S.bf16_bits_to_f32(oracle.f64_to_bf16_bits(X @ W.T))
        assert rel_frobenius(got[r0:r1], ref) <= 2e-3
        assert np.mean(got[r0:r1] == ref) > 0.99


@pytest.mark.parametrize("sizes,k,I", [([130, 0, 7], 256, 256), ([200] * 40, 512, 512)])
def test_mx_gemm_swiglu_pow2_h(sizes, k, I):
    import fp8_block_scaled_affinity_b200 as moe
    need_gpu()
    out, out_sf, res, off = _run_mx(sizes, k, 2 * I, moe.MOE_EPI_SWIGLU_QUANT, seed=len(sizes) + k)
    q = out.cpu().numpy()
    e = out_sf.cpu().numpy().T.astype(np.int32) - 127
    for g, (X, W) in enumerate(res):
        r0, r1 = off[g], off[g + 1]
        if r1 == r0:
            continue
        ga = X @ W[:I].T
        up = X @ W[I:].T
        h32 = ((ga / (1.0 + np.exp(-ga))) * up).astype(np.float32)
        hq, he = oracle.quant_act_1x128_pow2(h32)
        # exponents: equal unless the tile's amax sits on a power-of-two
        # boundary (fp32 accumulation order); codes one E4M3 step at most
        assert np.abs(e[r0:r1] - he).max() <= 1
        assert np.mean(e[r0:r1] == he) > 0.99
        same_e = np.repeat(e[r0:r1] == he, 128, axis=1)
        step = np.abs(_rank(q[r0:r1]) - _rank(hq))
        assert step[same_e].max() <= 1
        assert (step[same_e] == 0).mean() > 0.999
    assert np.all(q[off[-1]:] == 0xEE)


def test_quant_permute_ue8m0_bit_exact():
    import fp8_block_scaled_affinity_b200 as moe
    need_gpu()
    rng = np.random.default_rng(21)
    T, N, K, d = 300, 32, 6, 7168
    x = S.host_normal_bf16(rng, (T, d), 1.0)
    idx = np.stack([rng.choice(N, K, replace=False) for _ in range(T)]).astype(np.int32)
    counts = np.bincount(idx.ravel(), minlength=N).astype(np.int32)
    shape = moe.make_shape(T, d, N, 4, 4, K, 256, 0.001)
    R = T * K + T
    xq = torch.empty((R, d), dtype=torch.uint8, device=DEV)
    xsf = torch.empty((d // 128, R), dtype=torch.uint8, device=DEV)
    off = torch.empty(N + 2, dtype=torch.int32, device=DEV)
    rop = torch.empty((T, K), dtype=torch.int32, device=DEV)
    ws = torch.empty((moe.moe_permute_workspace_size(shape),), dtype=torch.uint8, device=DEV)
    moe.moe_quant_permute_ue8m0(shape, bf16_dev(x), to_dev(idx), to_dev(counts), xq, xsf, off,
                                rop, ws)
    torch.cuda.synchronize()
    q_o, e_o = oracle.quant_act_1x128_pow2(x)
    off_o, rop_o = oracle.permute_layout(idx, counts, N)
    assert np.array_equal(off.cpu().numpy(), off_o) and np.array_equal(rop.cpu().numpy(), rop_o)
    src = np.empty(R, np.int64)
    src[rop_o.ravel()] = np.repeat(np.arange(T), K)
    src[T * K:] = np.arange(T)
    assert np.array_equal(xq.cpu().numpy(), q_o[src])
    assert np.array_equal(xsf.cpu().numpy().T.astype(np.int32) - 127, e_o[src])


def _mx_layer(cfg_name, sample, seed_tokens=None):
    import fp8_block_scaled_affinity_b200 as moe
    from gpu_util import expert_bf16, host_bits
    cfg = S.CONFIGS[cfg_name]
    inp = S.make_layer_inputs_host(cfg, 0)
    shape = moe.make_shape(cfg.T, cfg.d, cfg.n_routed, cfg.n_groups, cfg.topk_groups, cfg.topk,
                           cfg.inter, cfg.gamma)
    layer = moe.MoeLayer(shape, bf16_dev(inp["router_w"]), to_dev(inp["bias"]), device=DEV,
                         scales="ue8m0")
    for e in range(cfg.n_routed + 1):
        layer.set_expert(e, *expert_bf16(cfg, e))
    off = None if inp["logit_offset"] is None else to_dev(inp["logit_offset"])
    y = layer.forward(bf16_dev(inp["x"]), logit_offset=off)
    torch.cuda.synchronize()
    assert layer.status() == 0
    cache = {}

    def experts(e):
        if e not in cache:
            cache[e] = oracle.quantized_expert_pow2(*(host_bits(w) for w in expert_bf16(cfg, e)))
        return cache[e]
    ref = oracle.layer_forward(inp["x"], inp["router_w"], inp["bias"], cfg.n_groups,
                               cfg.topk_groups, cfg.topk, experts,
                               logit_offset=inp["logit_offset"], tokens=sample, scales="pow2")
    assert np.array_equal(layer.topk_idx.cpu().numpy(), ref["topk_idx"])
    assert np.array_equal(layer.expert_counts.cpu().numpy(), ref["counts"])
    got = S.bf16_bits_to_f32(host_bits(y))[sample].astype(np.float64)
    exp = S.bf16_bits_to_f32(ref["y"]).astype(np.float64)
    fro = rel_frobenius(got, exp)
    tok = np.linalg.norm(got - exp, axis=1) / np.maximum(np.linalg.norm(exp, axis=1), 1e-30)
    print({"case": f"ue8m0 layer {cfg_name}", "tokens": len(sample), "rel_frobenius": fro,
           "worst_token_rel": float(tok.max())})
    assert fro <= 2e-3 and tok.max() <= 1e-2


def test_mx_layer_tiny_all_tokens():
    need_gpu()
    _mx_layer("tiny", np.arange(256))


def test_mx_layer_skewed_batch_sampled():
    need_gpu()
    _mx_layer("skewed", np.sort(np.random.default_rng(5).choice(16384, 512, replace=False)))
