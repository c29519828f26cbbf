"""Expert-parallel dispatch / combine driven by ep_forward over two gloo
ranks on the CPU ("DeepSeek-V3 Technical Report" notes page, section
"DualPipe": all-to-all dispatch and combine).  Each rank's stages are the
oracle restatement of tests/ep_oracle_stages.py (no GPU here); the test
checks the exchange logic of ep_forward (counts, row splits, the reversed
splits of the combine, the summed expert load of the bias update) against
the single-process oracle layer on every rank's batch."""
import os

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import synthetic as S

HERE = os.path.dirname(os.path.abspath(__file__))


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, os.path.dirname(HERE))
    sys.path.insert(0, HERE)
    import torch.distributed as dist
    import oracle
    from ep_oracle_stages import OracleEpStages
    from fp8_block_scaled_affinity_b200.ep import ep_forward
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        cfg = S.CONFIGS["tiny"]
        inp = S.make_layer_inputs_host(cfg, 0)
        T = 48
        cache = {}

        def experts(e):
            if e not in cache:
                cache[e] = oracle.quantized_expert(*S.host_expert_weights(cfg, e))
            return cache[e]
        results = []
        bias = inp["bias"].copy()
        for step in range(2):
            x = S.make_layer_inputs_host(cfg, 1 + world * step + rank)["x"][:T]
            st = OracleEpStages(cfg, rank, world, inp["router_w"], bias, experts, x)
            y = ep_forward(st, torch.from_numpy(x.view(np.int16)), update_bias=True)
            ref = oracle.layer_forward(x, inp["router_w"], bias, cfg.n_groups, cfg.topk_groups,
                                       cfg.topk, experts)
            got = y.numpy().view(np.uint16)
            results.append((bool(np.array_equal(got, ref["y"])),
                            float(np.abs(S.bf16_bits_to_f32(got) -
                                         S.bf16_bits_to_f32(ref["y"])).max())))
            bias = st.bias
        q.put((rank, results, bias.tolist()))
    finally:
        dist.destroy_process_group()


def test_ep_forward_two_gloo_ranks_match_the_oracle():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29600 + os.getpid() % 300
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(2):
        rank, res, bias = q.get(timeout=600)
        out[rank] = (res, bias)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in range(2):
        for equal, maxdiff in out[rank][0]:
            # the same FP64 sums grouped per destination: equal after the
            # bf16 rounding except where the grouping moves a rounding tie
            assert equal or maxdiff <= 2.0 ** -6, (rank, maxdiff)
    # both ranks carry the same bias: the update saw the summed load
    assert out[0][1] == out[1][1]
    # and it equals the update from the load of both ranks' batches together
    import oracle
    cfg = S.CONFIGS["tiny"]
    inp = S.make_layer_inputs_host(cfg, 0)
    b = inp["bias"].copy()
    for step in range(2):
        xs = [S.make_layer_inputs_host(cfg, 1 + 2 * step + r)["x"][:48] for r in range(2)]
        c = sum(oracle.route(x, inp["router_w"], b, cfg.n_groups, cfg.topk_groups,
                             cfg.topk)["counts"] for x in xs)
        b = oracle.update_bias(c, b, 96, cfg.topk, cfg.gamma)
    assert np.array_equal(np.array(out[0][1], np.float32).view(np.uint32), b.view(np.uint32))
