"""Host-side checks that need no GPU: the C library loads and exports every
entry point its header declares; argument validation rejects bad shapes
before any CUDA call; workspace sizes; the benchmark's multi-rank timing
aggregation over gloo (world size 2)."""
import ctypes
import os
import re
import socket

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def moe():
    import __graft_entry__
    __graft_entry__.build()
    import fp8_block_scaled_affinity_b200 as m
    return m


def declared_functions():
    text = open(os.path.join(ROOT, "include", "moefp8.h")).read()
    return re.findall(r"MOE_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def test_header_declares_the_seven_stages(moe):
    names = set(declared_functions())
    for n in ("moe_route", "fp8_quant_act_1x128", "fp8_quant_w_128x128", "moe_permute",
              "moe_grouped_gemm_fp8", "moe_combine", "moe_update_bias"):
        assert n in names


def test_library_exports_every_declared_symbol(moe):
    L = ctypes.CDLL(moe._lib.LIB_PATH)
    names = declared_functions()
    assert len(names) >= 16
    for n in names:
        assert hasattr(L, n), n
    assert moe.moe_version() == 100


def test_gemm_form_query(moe, monkeypatch):
    """moe_grouped_gemm_form: invalid arguments give 0; single CTAs unless
    MOEFP8_GEMM_PAIR=1; never a pair where the output width is not a
    multiple of 256."""
    f = moe.moe_grouped_gemm_form
    assert f(0, 128, 256, moe.MOE_EPI_F32) == 0
    assert f(1, 128, 200, moe.MOE_EPI_F32) == 0
    assert f(1, 128, 384, moe.MOE_EPI_SWIGLU_QUANT) == 0
    assert f(1, 128, 256, 9) == 0
    monkeypatch.setenv("MOEFP8_GEMM_PAIR", "0")
    assert f(1, 4096, 2048, moe.MOE_EPI_BF16) == 1
    monkeypatch.delenv("MOEFP8_GEMM_PAIR")
    assert f(257, 36864 + 4096, 4096, moe.MOE_EPI_SWIGLU_QUANT) == 1
    assert f(257, 1152 + 128, 7168, moe.MOE_EPI_F32) == 1
    assert f(1, 4096, 2048, moe.MOE_EPI_BF16) == 1
    assert f(1, 4096, 384, moe.MOE_EPI_F32) == 1
    monkeypatch.setenv("MOEFP8_GEMM_PAIR", "1")
    assert f(1, 4096, 384, moe.MOE_EPI_F32) == 1
    # pairs where the device allows them (none without a GPU)
    assert f(1, 4096, 2048, moe.MOE_EPI_BF16) in (1, 2)


def test_status_strings(moe):
    assert moe.status_string(0) == "ok"
    assert "workspace" in moe.status_string(-6)


def test_validation_before_any_cuda_call(moe):
    L = moe.lib()
    # activation quantiser: cols not a multiple of 128
    assert L.fp8_quant_act_1x128(None, 4, 100, None, None, 0, None, None) == -2
    assert L.fp8_quant_act_1x128(None, 0, 128, None, None, 0, None, None) == 0
    assert L.fp8_quant_act_1x128(None, 4, 128, None, None, 0, None, None) == -1
    assert L.fp8_quant_w_128x128(None, 100, 128, None, None, None, None) == -2
    # routing shapes
    bad = [moe.make_shape(4, 128, 10, 3, 1, 2, 128),   # N_r % G
           moe.make_shape(4, 128, 16, 4, 1, 5, 128),   # M * n_g < K
           moe.make_shape(4, 128, 16, 4, 5, 2, 128),   # M > G
           moe.make_shape(4, 128, 64, 64, 1, 1, 128),  # G > 32
           moe.make_shape(4, 128, 16, 4, 2, 33, 128)]  # K > 32
    for s in bad:
        assert L.moe_route(ctypes.byref(s), None, None, None, None, None, None, None, None, 0,
                           None, None) == -3
    s = moe.make_shape(4, 100, 16, 4, 2, 4, 128)
    assert L.moe_route(ctypes.byref(s), None, None, None, None, None, None, None, None, 0,
                       None, None) == -2
    # grouped GEMM arguments
    assert L.moe_grouped_gemm_fp8(1, 1, 1, 1, 1, 100, 1, 1, 128, 0, 1, None, None, None) == -2
    assert L.moe_grouped_gemm_fp8(1, 1, 1, 1, 1, 128, 1, 1, 128, 9, 1, None, None, None) == -7
    assert L.moe_grouped_gemm_fp8(1, 1, 1, 1, 1, 128, 1, 1, 128, 2, 1, None, None, None) == -2
    assert L.moe_grouped_gemm_fp8(0, 1, 1, 1, 1, 128, 1, 1, 128, 0, 1, None, None, None) == -2
    assert L.moe_grouped_gemm_fp8(1, None, 1, 1, 1, 128, 1, 1, 128, 0, 1, None, None, None) == -1
    # fused quantise + permute: missing x, misaligned x, missing workspace
    s = moe.make_shape(4, 128, 16, 4, 2, 4, 128)
    sp = ctypes.byref(s)
    assert L.moe_quant_permute(sp, None, 16, 16, 16, 16, 16, 16, 16, 1 << 20, None, None) == -1
    assert L.moe_quant_permute(sp, 8, 16, 16, 16, 16, 16, 16, 16, 1 << 20, None, None) == -5
    assert L.moe_quant_permute(sp, 16, 16, 16, 16, 16, 16, 16, None, 0, None, None) == -6


def test_workspace_sizes(moe):
    T, d, N, K, I = 4096, 7168, 256, 8, 2048
    s = moe.make_shape(T, d, N, 8, 4, K, I)
    R = T * K + T
    assert moe.moe_route_workspace_size(s) >= T * N * 4
    assert moe.moe_permute_workspace_size(s) >= (T // 64) * N * 4
    ws = moe.moe_layer_workspace_size(s)
    # permuted codes + scales, h codes + scales, fp32 expert outputs (x is
    # quantised straight into its permuted rows: no unpermuted copy)
    need = R * d + R * d // 32 + R * I + R * I // 32 + R * d * 4
    scratch = moe.moe_route_workspace_size(s) + moe.moe_permute_workspace_size(s)
    assert need + scratch <= ws <= need + scratch + 64 * 1024
    assert moe.moe_layer_host_workspace_size(s) >= ws + 2 * T * d * 2
    assert moe.moe_layer_workspace_size(moe.make_shape(4, 128, 10, 3, 1, 2, 128)) == 0


def test_algorithmic_counts_prefill():
    import bench
    import synthetic as S
    cfg = S.CONFIGS["prefill"]
    counts = np.full(cfg.n_routed, cfg.T * cfg.topk // cfg.n_routed)
    a = bench.algorithmic_counts(cfg, counts)
    assert a["rows"] == 36864 and a["touched"] == 257
    # 2*3*d*I flops per row
    assert a["layer_flops"] == pytest.approx(36864 * 6 * 7168 * 2048)
    # touched FP8 weights dominate the layer's bytes: 257 * 3 * d * I
    assert a["layer_bytes"] == pytest.approx(257 * 3 * 7168 * 2048 + 2 * 4096 * 7168 * 2,
                                             rel=1e-3)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        m = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        bench.barrier(world)
        q.put((rank, m))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert got == [(0, 15.0), (1, 15.0)]


def test_reference_arm_json_line_on_cpu():
    """`bench.py --impl reference` (the oracle on the host cores) prints one
    JSON line with the contract's keys, on the same workload name as the
    GPU arm."""
    import json
    import subprocess
    import sys
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["config"]["workload"] == "moe_layer_tiny"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert line["higher_is_better"] is True
