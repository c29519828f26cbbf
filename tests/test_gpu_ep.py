"""Expert-parallel dispatch / combine kernels on one GPU ("DeepSeek-V3
Technical Report" notes page, section "DualPipe": all-to-all dispatch and
combine of FP8 activations).  P ranks are emulated in one process: each
rank's stages run on the GPU through the library, and each all-to-all is a
local copy that hands rank p's rows for rank q to rank q (the real
multi-process exchange is NCCL's all_to_all_single, driven by ep_forward and
tested over gloo on the CPU).  Checked: the dispatch rows byte for byte
against the oracle's restatement of the row format, routing and counts bit
for bit, and every rank's y against the oracle layer on that rank's batch."""
import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from ep_oracle_stages import OracleEpStages
from gpu_util import DEV, bf16_dev, expert_bf16, host_bits, need_gpu, rel_frobenius, to_dev

pytestmark = pytest.mark.gpu


def _emulated_forward(layers, xs):
    """ep_forward's stages for all ranks in lockstep, exchanges as copies."""
    P = len(layers)
    sends = [l.route_and_pack(x) for l, x in zip(layers, xs)]
    offs = [np.concatenate([[0], np.cumsum(c)]) for _, c in sends]
    recv, src_off = [], []
    for q in range(P):
        parts = [sends[p][0][offs[p][q]:offs[p][q + 1]] for p in range(P)]
        recv.append(torch.cat(parts) if parts else None)
        src_off.append(np.concatenate([[0], np.cumsum([sends[p][1][q] for p in range(P)])]))
    backs = [layers[q].experts(recv[q], int(src_off[q][-1])) for q in range(P)]
    ys = []
    for p in range(P):
        parts = [backs[q][src_off[q][p]:src_off[q][p + 1]] for q in range(P)]
        ys.append(layers[p].shared_and_combine(xs[p], torch.cat(parts)))
    return ys, sends


@pytest.mark.parametrize("cfg_name,P,T", [("tiny", 4, 64), ("tiny", 2, 100),
                                          ("prefill_e16", 8, 128)])
def test_emulated_expert_parallel_layer(cfg_name, P, T):
    import fp8_block_scaled_affinity_b200 as moe
    from fp8_block_scaled_affinity_b200.ep import EpMoeLayer
    need_gpu()
    cfg = S.CONFIGS[cfg_name]
    inp = S.make_layer_inputs_host(cfg, 0)
    shape = moe.make_shape(T, cfg.d, cfg.n_routed, cfg.n_groups, cfg.topk_groups, cfg.topk,
                           cfg.inter, cfg.gamma)
    rw, bias = bf16_dev(inp["router_w"]), to_dev(inp["bias"])
    layers = [EpMoeLayer(shape, q, P, rw, bias.clone(), device=DEV) for q in range(P)]
    for e in range(cfg.n_routed + 1):
        w = expert_bf16(cfg, e)
        for l in layers:
            l.set_expert(e, *w)
    xs_bits = [S.make_layer_inputs_host(cfg, 1 + q)["x"][:T] for q in range(P)]
    ys, sends = _emulated_forward(layers, [bf16_dev(x) for x in xs_bits])
    torch.cuda.synchronize()
    cache = {}

    def experts(e):
        if e not in cache:
            cache[e] = oracle.quantized_expert(*(host_bits(w) for w in expert_bf16(cfg, e)))
        return cache[e]
    for q in range(P):
        assert layers[q].dev_status.item() == 0
        ref_st = OracleEpStages(cfg, q, P, inp["router_w"], inp["bias"], experts, xs_bits[q])
        ref_buf, ref_counts = ref_st.route_and_pack(None)
        assert sends[q][1] == ref_counts
        n = sum(ref_counts)
        assert np.array_equal(sends[q][0][:n].cpu().numpy(), ref_buf.numpy()[:n])
        ref = oracle.layer_forward(xs_bits[q], inp["router_w"], inp["bias"], cfg.n_groups,
                                   cfg.topk_groups, cfg.topk, experts)
        assert np.array_equal(layers[q].topk_idx.cpu().numpy(), ref["topk_idx"])
        got = S.bf16_bits_to_f32(host_bits(ys[q])).astype(np.float64)
        exp = S.bf16_bits_to_f32(ref["y"]).astype(np.float64)
        assert rel_frobenius(got, exp) <= 2e-3
        tok = np.linalg.norm(got - exp, axis=1) / np.linalg.norm(exp, axis=1)
        assert tok.max() <= 5e-2


def test_ep_kernels_reject_bad_arguments():
    import fp8_block_scaled_affinity_b200 as moe
    need_gpu()
    shape = moe.make_shape(4, 256, 16, 4, 2, 4, 256, 0.001)
    z = torch.zeros(64, dtype=torch.int32, device=DEV)
    ws = torch.empty((moe.moe_ep_workspace_size(shape, 4, 0),), dtype=torch.uint8, device=DEV)
    with pytest.raises(moe.MoeError) as e:
        moe.moe_ep_dispatch_plan(shape, 3, z, z, z, z, ws)  # 16 experts on 3 ranks
    assert e.value.status == -7
