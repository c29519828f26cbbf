"""The no-allocation permutation entry point (moe_permute_static_ws).

It serves callers that cannot allocate device memory while they run, for
example a serving loop whose memory budget is fixed at start-up or a host
framework that owns all device memory through its own pool: they get the
permutation without passing a workspace, because the scratch lives in a
fixed device array inside the library.  Its results must equal those of
moe_permute (the entry point that takes a caller workspace) bit for bit:
the permutation is integer and byte work.  The calls go through the C ABI
with ctypes.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _case(T, N, K, d, seed):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.choice(N, K, replace=False) for _ in range(T)]).astype(np.int32)
    counts = np.bincount(idx.ravel(), minlength=N).astype(np.int32)
    xq = rng.integers(0, 256, size=(T, d), dtype=np.uint8)
    xs = rng.uniform(0.001, 1.0, size=(T, d // 128)).astype(np.float32)
    return {k: torch.from_numpy(v).to(DEV) for k, v in
            dict(idx=idx, counts=counts, xq=xq, xs=xs).items()}


def _outputs(T, N, K, d):
    R = T * K + T
    return (torch.full((R, d), 0xAB, dtype=torch.uint8, device=DEV),
            torch.full((d // 128, R), -7.0, dtype=torch.float32, device=DEV),
            torch.full((N + 2,), -1, dtype=torch.int32, device=DEV),
            torch.full((T, K), -1, dtype=torch.int32, device=DEV))


def _call_c(name, shape, inp, outs, ws=None):
    import fp8_block_scaled_affinity_b200 as moe
    L = moe.lib()
    st = torch.cuda.current_stream().cuda_stream
    args = [ctypes.byref(shape), inp["idx"].data_ptr(), inp["counts"].data_ptr(),
            inp["xq"].data_ptr(), inp["xs"].data_ptr()] + [o.data_ptr() for o in outs]
    if ws is not None:
        args += [ws.data_ptr(), ws.numel()]
    rc = getattr(L, name)(*args, None, st)
    assert rc == 0, moe.status_string(rc)


def test_static_workspace_entry_point_matches_workspace_entry_point():
    import fp8_block_scaled_affinity_b200 as moe
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    # two calls in a row on different shapes: the second must not see the
    # first call's scratch contents
    for T, N, K, d, seed in [(1000, 256, 8, 1024, 1), (257, 16, 4, 512, 2)]:
        shape = moe.make_shape(T, d, N, 1, 1, K, 128)
        inp = _case(T, N, K, d, seed)
        ref = _outputs(T, N, K, d)
        ws = torch.empty((moe.moe_permute_workspace_size(shape),), dtype=torch.uint8, device=DEV)
        _call_c("moe_permute", shape, inp, ref, ws)
        got = _outputs(T, N, K, d)
        _call_c("moe_permute_static_ws", shape, inp, got)
        torch.cuda.synchronize()
        for a, b in zip(got, ref):
            assert torch.equal(a.view(torch.uint8) if a.dtype == torch.uint8 else a.view(torch.int32),
                               b.view(torch.uint8) if b.dtype == torch.uint8 else b.view(torch.int32))


def test_static_workspace_entry_point_rejects_shapes_beyond_its_limit():
    import fp8_block_scaled_affinity_b200 as moe
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    L = moe.lib()
    # ceil(T/64) * N_r = 1025 * 256 > 262144
    shape = moe.make_shape(65600, 128, 256, 8, 4, 8, 128)
    rc = L.moe_permute_static_ws(ctypes.byref(shape), 1, 1, 16, 16, 16, 16, 1, 1, None, None)
    assert rc == -9
    assert "fixed scratch" in moe.status_string(rc)
