"""Redundant experts on the GPU (618zxw.cn news article on DeepSeek-V3:
copies of the most loaded experts for inference load balance): the group
table of the copies matches the oracle bit for bit, and the layer computed
with the copies (each a group of the indexed grouped GEMM sharing its
expert's weights) gives the same bits as the layer without them."""
import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from gpu_util import DEV, bf16_dev, need_gpu, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n_extra", [1, 12, 40])
def test_layer_with_redundant_copies_is_bit_identical(n_extra):
    import fp8_block_scaled_affinity_b200 as moe
    need_gpu()
    cfg = S.CONFIGS["tiny"]
    inp = S.make_layer_inputs_host(cfg, 0)
    shape = moe.make_shape(cfg.T, cfg.d, cfg.n_routed, cfg.n_groups, cfg.topk_groups, cfg.topk,
                           cfg.inter, cfg.gamma)
    layer = moe.MoeLayer(shape, bf16_dev(inp["router_w"]), to_dev(inp["bias"]), device=DEV)
    for e in range(cfg.n_routed + 1):
        layer.set_expert(e, *(bf16_dev(m) for m in S.host_expert_weights(cfg, e)))
    # a skewed load: a Zipf prior on the logits makes a few experts hot
    offset = to_dev(S.zipf_logit_offset(cfg.n_routed, 1.2))
    x = bf16_dev(inp["x"])
    y_ref = layer.forward(x, logit_offset=offset).clone()
    torch.cuda.synchronize()

    T, d, I, N, K = cfg.T, cfg.d, cfg.inter, cfg.n_routed, cfg.topk
    R = T * K + T
    counts = layer.expert_counts.cpu().numpy()
    offsets = layer.expert_offsets  # from the forward pass above
    rep, slots = moe.moe_plan_redundant_experts(counts, n_extra)
    first = np.concatenate([[0], np.cumsum(rep)[:-1]]).astype(np.int32)
    G = N + n_extra + 1
    so = torch.empty(G + 1, dtype=torch.int32, device=DEV)
    sw = torch.empty(G, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    moe.moe_split_groups(shape, offsets, to_dev(rep), to_dev(slots), to_dev(first), n_extra, so,
                         sw, status)
    so_ref, sw_ref = oracle.split_groups(offsets.cpu().numpy(), rep)
    assert np.array_equal(so.cpu().numpy(), so_ref) and np.array_equal(sw.cpu().numpy(), sw_ref)

    # the layer's stages again, the expert GEMMs over the copies' groups
    xq = torch.empty((R, d), dtype=torch.uint8, device=DEV)
    xs = torch.empty((d // 128, R), dtype=torch.float32, device=DEV)
    hq = torch.empty((R, I), dtype=torch.uint8, device=DEV)
    hs = torch.empty((I // 128, R), dtype=torch.float32, device=DEV)
    o = torch.empty((R, d), dtype=torch.float32, device=DEV)
    y = torch.empty_like(x)
    pws = torch.empty((moe.moe_permute_workspace_size(shape),), dtype=torch.uint8, device=DEV)
    moe.moe_quant_permute(shape, x, layer.topk_idx, layer.expert_counts, xq, xs,
                          layer.expert_offsets, layer.row_of_pair, pws)
    moe.moe_grouped_gemm_fp8_indexed(G, so, sw, N + 1, R, xq, xs, d, layer.w13,
                                     layer.w13_scales, 2 * I, moe.MOE_EPI_SWIGLU_QUANT, hq, hs,
                                     status)
    moe.moe_grouped_gemm_fp8_indexed(G, so, sw, N + 1, R, hq, hs, I, layer.w2, layer.w2_scales, d,
                                     moe.MOE_EPI_F32, o, None, status)
    moe.moe_combine(shape, o, layer.expert_offsets, layer.row_of_pair, layer.topk_gate, y)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
    # the largest group of routed rows shrinks to the planner's bound
    sizes = np.diff(so_ref)[:-1]
    assert sizes.max() == max(-(-int(c) // int(r)) for c, r in zip(counts, rep))
