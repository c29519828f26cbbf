"""GPU parity of the tcgen05 grouped FP8 GEMM against the oracle's FP64
matmul over dequantised values ("DeepSeek-V3 Technical Report" notes page,
section "FP8 mixed precision training": FP8 GEMM inputs with 1x128 / 128x128
scales, FP32 accumulation promoted every 128 elements of K).

Tolerances: with FP32 accumulation of FP8 products and per-block promotion,
the relative error of an output is a few fp32 rounding steps (about 1e-6);
1e-5 relative Frobenius is used for fp32 outputs.  bf16 outputs are compared
after both sides round to bf16 (2e-3, the layer's output bound).

Every test runs twice: with single CTAs (the library's default) and with
CTA pairs (cta_group::2, selected with MOEFP8_GEMM_PAIR=1 where the output
width allows it)."""
import os

import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from gpu_util import DEV, bf16_dev, need_gpu, rel_frobenius, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, params=["pair", "single"])
def cta_mode(request, monkeypatch):
    """Select the GEMM kernel form for the test (read by the library at every
    call)."""
    monkeypatch.setenv("MOEFP8_GEMM_PAIR", "1" if request.param == "pair" else "0")
    return request.param


def _quant_gpu(xbits):
    import fp8_block_scaled_affinity_b200 as moe
    rows, cols = xbits.shape
    q = torch.empty((rows, cols), dtype=torch.uint8, device=DEV)
    s = torch.empty((cols // 128, rows), dtype=torch.float32, device=DEV)
    moe.fp8_quant_act_1x128(bf16_dev(xbits), q, s, True)
    return q, s


def _quant_w_gpu(wbits):
    import fp8_block_scaled_affinity_b200 as moe
    rows, cols = wbits.shape
    q = torch.empty((rows, cols), dtype=torch.uint8, device=DEV)
    s = torch.empty((rows // 128, cols // 128), dtype=torch.float32, device=DEV)
    moe.fp8_quant_w_128x128(bf16_dev(wbits), q, s)
    return q, s


def run_grouped(sizes, k, n, epilogue, seed, pad_rows=0, outliers=False, inputs=None):
    """Random A rows split into groups of `sizes`, one weight matrix per group.
    Returns (gpu_out, oracle_results_per_group, offsets, extras)."""
    import fp8_block_scaled_affinity_b200 as moe
    rng = np.random.default_rng(seed)
    G = len(sizes)
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    R = int(off[-1]) + pad_rows
    va = rng.standard_normal((R, k)).astype(np.float32)
    if outliers:
        va *= np.where(rng.random((R, k)) < 0.001, 100.0, 1.0).astype(np.float32)
    a = S.f32_to_bf16_bits(va)
    w = S.host_normal_bf16(rng, (G * n, k), 0.05)
    if inputs is not None:
        inputs.update(a=a, w=w)
    aq, as_ = _quant_gpu(a)
    wq, ws = _quant_w_gpu(w)
    if epilogue == moe.MOE_EPI_SWIGLU_QUANT:
        out = torch.full((R, n // 2), 0xEE, dtype=torch.uint8, device=DEV)
        out_s = torch.full((n // 2 // 128, R), -1.0, dtype=torch.float32, device=DEV)
    elif epilogue == moe.MOE_EPI_F32:
        out = torch.full((R, n), float("nan"), dtype=torch.float32, device=DEV)
        out_s = None
    else:
        out = torch.full((R, n), float("nan"), dtype=torch.bfloat16, device=DEV)
        out_s = None
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    moe.moe_grouped_gemm_fp8(G, to_dev(off), R, aq, as_, k, wq, ws, n, epilogue, out, out_s,
                             status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    # oracle, from the same bf16 inputs
    qa_o, sa_o = oracle.quant_act_1x128(a)
    res = []
    for g in range(G):
        r0, r1 = off[g], off[g + 1]
        wg = w[g * n:(g + 1) * n]
        if epilogue == moe.MOE_EPI_SWIGLU_QUANT:
            I = n // 2
            w1q, w1s = oracle.quant_w_128x128(wg[:I])
            w3q, w3s = oracle.quant_w_128x128(wg[I:])
            X = oracle.dequant_act(qa_o[r0:r1], sa_o[r0:r1])
            ga = X @ oracle.dequant_w(w1q, w1s).T
            up = X @ oracle.dequant_w(w3q, w3s).T
            h32 = ((ga / (1.0 + np.exp(-ga))) * up).astype(np.float32)
            res.append((h32,) + oracle.quant_act_1x128(h32) if r1 > r0 else None)
        else:
            wq_o, ws_o = oracle.quant_w_128x128(wg)
            res.append(oracle.gemm_blockscaled(qa_o[r0:r1], sa_o[r0:r1], wq_o, ws_o))
    return out, out_s, res, off


def _check_dense(out, res, off, epilogue):
    import fp8_block_scaled_affinity_b200 as moe
    if epilogue == moe.MOE_EPI_F32:
        got = out.cpu().numpy()
    else:
        got = S.bf16_bits_to_f32(out.cpu().view(torch.int16).numpy().view(np.uint16))
    for g, ref in enumerate(res):
        r0, r1 = off[g], off[g + 1]
        if r1 == r0:
            continue
        if epilogue == moe.MOE_EPI_F32:
            assert rel_frobenius(got[r0:r1], ref) <= 1e-5, g
        else:
            refb = S.bf16_bits_to_f32(oracle.f64_to_bf16_bits(ref))
            assert rel_frobenius(got[r0:r1], refb) <= 2e-3, g
    # rows outside every group stay untouched
    if got.shape[0] > off[-1]:
        assert np.all(np.isnan(got[off[-1]:]))


@pytest.mark.parametrize("sizes,k,n", [([1], 128, 128), ([300], 512, 256), ([256], 256, 128),
                                       ([257, 0, 5, 16, 17], 384, 256),
                                       ([40] * 9 + [600], 1024, 384),
                                       ([130, 1, 600, 255, 256, 17, 64, 33], 256, 512),
                                       # token boxes of exactly 16, 32, 64 rows and just above
                                       ([16, 32, 64, 65, 48, 96, 144, 160, 192], 384, 768)])
def test_grouped_fp32_output(sizes, k, n):
    import fp8_block_scaled_affinity_b200 as moe
    need_gpu()
    out, _, res, off = run_grouped(sizes, k, n, moe.MOE_EPI_F32, seed=sum(sizes) + k, pad_rows=3)
    _check_dense(out, res, off, moe.MOE_EPI_F32)


def test_bf16_output_with_outliers():
    import fp8_block_scaled_affinity_b200 as moe
    need_gpu()
    out, _, res, off = run_grouped([333], 1024, 512, moe.MOE_EPI_BF16, seed=5, outliers=True)
    _check_dense(out, res, off, moe.MOE_EPI_BF16)


@pytest.mark.parametrize("sizes,k,I", [([1], 128, 128), ([130, 0, 7], 256, 256),
                                       ([128, 129, 64], 512, 128)])
def test_swiglu_quant_epilogue(sizes, k, I):
    import fp8_block_scaled_affinity_b200 as moe
    need_gpu()
    out, out_s, res, off = run_grouped(sizes, k, 2 * I, moe.MOE_EPI_SWIGLU_QUANT,
                                       seed=len(sizes) * 7 + k)
    q = out.cpu().numpy()
    s = out_s.cpu().numpy().T  # -> [rows, I/128]
    table = oracle.e4m3_decode_table()
    for g, ref in enumerate(res):
        r0, r1 = off[g], off[g + 1]
        if ref is None:
            continue
        h32, hq_ref, hs_ref = ref
        # scales: amax of h over 128 features; fp32 accumulation order only
        assert np.allclose(s[r0:r1], hs_ref, rtol=1e-5, atol=0)
        # codes: equal except rare one-step flips at rounding boundaries
        same = q[r0:r1] == hq_ref
        assert same.mean() > 0.999
        dq = table[q[r0:r1]] * np.repeat(s[r0:r1], 128, axis=1)
        assert rel_frobenius(dq, h32) <= 5e-2  # E4M3 itself: about 2.4% RMS
        dq_ref = table[hq_ref] * np.repeat(hs_ref, 128, axis=1)
        assert rel_frobenius(dq, dq_ref) <= 2e-3


def test_full_size_gemm_workload():
    """A 4096x7168 (1x128 scales, 0.1% x100 outliers) times B 7168x2048
    (128x128 scales), bf16 out: the GEMM-alone workload."""
    import fp8_block_scaled_affinity_b200 as moe
    need_gpu()
    cfg = S.GEMM_C2
    a, b = S.make_gemm_inputs_host(cfg)
    aq, as_ = _quant_gpu(a)
    bq, bs = _quant_w_gpu(b)
    off = to_dev(np.array([0, cfg.m], np.int32))
    out = torch.empty((cfg.m, cfg.n), dtype=torch.bfloat16, device=DEV)
    moe.moe_grouped_gemm_fp8(1, off, cfg.m, aq, as_, cfg.k, bq, bs, cfg.n, moe.MOE_EPI_BF16, out)
    torch.cuda.synchronize()
    got = S.bf16_bits_to_f32(out.cpu().view(torch.int16).numpy().view(np.uint16))
    qa, sa = oracle.quant_act_1x128(a)
    qb, sb = oracle.quant_w_128x128(b)
    # the same quantised operands on both sides
    assert np.array_equal(aq.cpu().numpy(), qa) and np.array_equal(bq.cpu().numpy(), qb)
    ref = S.bf16_bits_to_f32(oracle.f64_to_bf16_bits(oracle.gemm_blockscaled(qa, sa, qb, sb)))
    assert rel_frobenius(got, ref) <= 2e-3
    assert np.mean(got == ref) > 0.99


def test_gemm_rejects_bad_arguments():
    import fp8_block_scaled_affinity_b200 as moe
    need_gpu()
    z = torch.zeros(1024, dtype=torch.uint8, device=DEV)
    off = to_dev(np.array([0, 1], np.int32))
    for args, code in [((1, off, 1, z, z, 100, z, z, 128, 0, z), -2),
                       ((1, off, 1, z, z, 128, z, z, 128, 9, z), -7),
                       ((1, off, 1, z, z, 128, z, z, 256, 2, z, None), -1),  # no out_scales
                       ((1, off, 1, z, z, 128, z, z, 128, 2, z, z), -2)]:    # n % 256
        with pytest.raises(moe.MoeError) as e:
            moe.moe_grouped_gemm_fp8(*args)
        assert e.value.status == code


# ----------------------------------------------------------------------
# Many work items per CTA, compared element by element.
#
# The GEMM is persistent: one CTA (or CTA pair) per SM walks a strided list
# of (group, column tile, token tile) items, handing TMEM partial buffers,
# stage barriers and (SwiGLU) the alternating amax exchange over from item
# to item.  With 64 groups of 130-300 rows there are well over 2 x 148
# items, so every CTA runs several of them.

def _rank(codes):
    """Order-preserving integer of an E4M3 code (both zeros -> 0)."""
    c = codes.astype(np.int32)
    mag = c & 0x7F
    return np.where(c & 0x80, -mag, mag)


def _many_items_sizes(seed):
    return np.random.default_rng(seed).integers(130, 301, size=64).tolist()


@pytest.mark.parametrize("epilogue_name,n,k", [("f32", 2048, 512), ("swiglu", 4096, 512),
                                                ("f32", 768, 1024)])
def test_many_items_per_cta_element_wise(epilogue_name, n, k):
    import fp8_block_scaled_affinity_b200 as moe
    need_gpu()
    epi = moe.MOE_EPI_F32 if epilogue_name == "f32" else moe.MOE_EPI_SWIGLU_QUANT
    sizes = _many_items_sizes(seed=n + k)
    ctas = 2 if moe.moe_grouped_gemm_form(len(sizes), sum(sizes), n, epi) == 2 else 1
    tile_rows = 128 * ctas
    tile_cols = 256 if (epi == moe.MOE_EPI_SWIGLU_QUANT or n % 256 == 0) else 128
    items = sum((s + tile_rows - 1) // tile_rows for s in sizes) * (n // tile_cols)
    assert items > 2 * (148 // ctas)  # several items per CTA (pair)
    inp = {}
    out, out_s, res, off = run_grouped(sizes, k, n, epi, seed=n * 7 + k, pad_rows=5, inputs=inp)
    nkb = k // 128
    if epi == moe.MOE_EPI_F32:
        got = out.cpu().numpy().astype(np.float64)
        # every element: FP32 accumulation of 128 exact products per K block
        # (at most 127 roundings) and one promotion FMA per block, each
        # rounding at most one fp32 ulp (2^-23 relative, whatever the
        # rounding mode), so |got - exact| <= 2^-23 (128 + nkb + 2)
        # sum_k |a_k b_k| s_a s_b
        a, w = inp["a"], inp["w"]
        qa, sa = oracle.quant_act_1x128(a)
        for g, ref in enumerate(res):
            r0, r1 = off[g], off[g + 1]
            wq, ws = oracle.quant_w_128x128(w[g * n:(g + 1) * n])
            absum = np.abs(oracle.dequant_act(qa[r0:r1], sa[r0:r1])) @ \
                np.abs(oracle.dequant_w(wq, ws)).T
            bound = 2.0 ** -23 * (128 + nkb + 2) * absum
            err = np.abs(got[r0:r1] - ref)
            bad = err > bound
            assert not bad.any(), (g, int(bad.sum()), float(err.max()))
        assert np.all(np.isnan(got[off[-1]:]))
    else:
        q = out.cpu().numpy()
        s = out_s.cpu().numpy().T
        for g, ref in enumerate(res):
            r0, r1 = off[g], off[g + 1]
            h32, hq_ref, hs_ref = ref
            # scales: the same amax up to fp32 accumulation order
            assert np.allclose(s[r0:r1], hs_ref, rtol=1e-5, atol=0), g
            # codes: every one equal or one E4M3 step away (h at a rounding
            # boundary), and almost all equal
            step = np.abs(_rank(q[r0:r1]) - _rank(hq_ref))
            assert step.max() <= 1, (g, int(step.max()))
            assert (step == 0).mean() > 0.999, g
        # rows outside every group are not written
        assert np.all(q[off[-1]:] == 0xEE)
        assert np.all(s[off[-1]:] == -1.0)
