"""Failure detection on the GPU without a GPU fault.

A bounded wait inside a kernel that runs out must end the kernel with
MOE_DEV_TIMEOUT on the caller's status word, leave the CUDA context usable,
and let the next call run normally.  The failure is made on the host: the
environment variable MOEFP8_FAULT=gemm_producer makes the single-CTA grouped
GEMM's TMA producer withhold the loads of its first stage (so the MMA
issuer's wait on that stage can never finish), and MOEFP8_WAIT_LIMIT_NS
shortens every wait of the launch to 20 microseconds.  Nothing faults,
traps or hangs: the wait limit ends the wait, every role of the CTA sees
the abort flag, work already in flight is waited for, and TMEM is freed."""
import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from gpu_util import DEV, bf16_dev, need_gpu, rel_frobenius, to_dev

pytestmark = pytest.mark.gpu

MOE_DEV_TIMEOUT = 1


def _gemm_case(epilogue):
    import fp8_block_scaled_affinity_b200 as moe
    rng = np.random.default_rng(123)
    sizes = [300, 17, 256, 129]
    k, n = 1024, 512
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    R = int(off[-1])
    a = S.f32_to_bf16_bits(rng.standard_normal((R, k)).astype(np.float32))
    w = S.host_normal_bf16(rng, (len(sizes) * n, k), 0.05)
    aq = torch.empty((R, k), dtype=torch.uint8, device=DEV)
    as_ = torch.empty((k // 128, R), dtype=torch.float32, device=DEV)
    moe.fp8_quant_act_1x128(bf16_dev(a), aq, as_, True)
    wq = torch.empty((len(sizes) * n, k), dtype=torch.uint8, device=DEV)
    ws = torch.empty((len(sizes) * n // 128, k // 128), dtype=torch.float32, device=DEV)
    moe.fp8_quant_w_128x128(bf16_dev(w), wq, ws)
    if epilogue == moe.MOE_EPI_F32:
        out = torch.empty((R, n), dtype=torch.float32, device=DEV)
        out_s = None
    else:
        out = torch.empty((R, n // 2), dtype=torch.uint8, device=DEV)
        out_s = torch.empty((n // 256, R), dtype=torch.float32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)

    def call():
        moe.moe_grouped_gemm_fp8(len(sizes), to_dev(off), R, aq, as_, k, wq, ws, n, epilogue,
                                 out, out_s, status)
    return call, out, out_s, status, (a, w, off, n)


@pytest.mark.parametrize("epilogue_name", ["f32", "swiglu"])
def test_gemm_wait_runs_out_then_next_call_is_correct(epilogue_name, monkeypatch):
    import fp8_block_scaled_affinity_b200 as moe
    need_gpu()
    monkeypatch.setenv("MOEFP8_GEMM_PAIR", "0")  # the injection is for single CTAs
    epi = moe.MOE_EPI_F32 if epilogue_name == "f32" else moe.MOE_EPI_SWIGLU_QUANT
    call, out, out_s, status, (a, w, off, n) = _gemm_case(epi)
    # a normal call first
    call()
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    good = out.clone()
    good_s = None if out_s is None else out_s.clone()

    # the injected failure: the wait on the withheld stage runs out
    monkeypatch.setenv("MOEFP8_FAULT", "gemm_producer")
    monkeypatch.setenv("MOEFP8_WAIT_LIMIT_NS", "20000")
    out.zero_()
    call()
    torch.cuda.synchronize()  # returns: the kernel ended by itself
    assert int(status.item()) == MOE_DEV_TIMEOUT

    # the context is usable and the next call is correct
    monkeypatch.delenv("MOEFP8_FAULT")
    monkeypatch.delenv("MOEFP8_WAIT_LIMIT_NS")
    status.zero_()
    out.zero_()
    call()
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(out.view(torch.uint8), good.view(torch.uint8))
    if good_s is not None:
        assert torch.equal(out_s, good_s)
    if epi == moe.MOE_EPI_F32:
        qa, sa = oracle.quant_act_1x128(a)
        for g in range(len(off) - 1):
            wq, ws = oracle.quant_w_128x128(w[g * n:(g + 1) * n])
            ref = oracle.gemm_blockscaled(qa[off[g]:off[g + 1]], sa[off[g]:off[g + 1]], wq, ws)
            assert rel_frobenius(out[off[g]:off[g + 1]].cpu().numpy(), ref) <= 1e-5
    # and plain torch work on the same context still runs
    x = torch.arange(1024, device=DEV, dtype=torch.float32)
    assert float(x.sum().item()) == 1023 * 1024 / 2


def test_layer_reports_timeout_and_recovers(monkeypatch):
    """The same injection inside a whole layer call: the W13 GEMM's wait runs
    out, the layer call returns (it does not hang), the status word says
    MOE_DEV_TIMEOUT, and the next layer call reproduces the first one."""
    import fp8_block_scaled_affinity_b200 as moe
    need_gpu()
    monkeypatch.setenv("MOEFP8_GEMM_PAIR", "0")
    cfg = S.CONFIGS["tiny"]
    inp = S.make_layer_inputs_host(cfg, 0)
    shape = moe.make_shape(cfg.T, cfg.d, cfg.n_routed, cfg.n_groups, cfg.topk_groups, cfg.topk,
                           cfg.inter, cfg.gamma)
    layer = moe.MoeLayer(shape, bf16_dev(inp["router_w"]), to_dev(inp["bias"]), device=DEV)
    for e in range(cfg.n_routed + 1):
        layer.set_expert(e, *(bf16_dev(m) for m in S.host_expert_weights(cfg, e)))
    x = bf16_dev(inp["x"])
    y0 = layer.forward(x).clone()
    assert layer.status() == 0
    monkeypatch.setenv("MOEFP8_FAULT", "gemm_producer")
    monkeypatch.setenv("MOEFP8_WAIT_LIMIT_NS", "20000")
    layer.forward(x)
    assert layer.status() == MOE_DEV_TIMEOUT
    monkeypatch.delenv("MOEFP8_FAULT")
    monkeypatch.delenv("MOEFP8_WAIT_LIMIT_NS")
    layer.dev_status.zero_()
    y1 = layer.forward(x)
    assert layer.status() == 0
    assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))
