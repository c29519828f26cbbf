"""Helpers shared by the GPU parity tests: device inputs built from the seeded
generator, calls through the C ABI, comparisons against the oracle."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synthetic as S

DEV = "cuda:0"


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def to_dev(a: np.ndarray, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.to(DEV)


def bf16_dev(bits: np.ndarray):
    """uint16 bf16 bit patterns -> torch.bfloat16 tensor on the GPU."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(DEV)


def host_bits(t) -> np.ndarray:
    """bf16 torch tensor -> uint16 numpy bit patterns on the host."""
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def rel_frobenius(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def shape_of(cfg: S.MoeConfig, T=None):
    import fp8_block_scaled_affinity_b200 as moe
    return moe.make_shape(cfg.T if T is None else T, cfg.d, cfg.n_routed, cfg.n_groups,
                          cfg.topk_groups, cfg.topk, cfg.inter, cfg.gamma)


def expert_bf16(cfg: S.MoeConfig, e: int):
    """(W1, W3, W2) bf16 on the GPU for expert e: host draws for the small
    workload, device draws for the full-size ones."""
    if cfg.d * cfg.inter <= 512 * 256:
        return tuple(bf16_dev(w) for w in S.host_expert_weights(cfg, e))
    return S.device_expert_weights(cfg, e, DEV)


class OracleExperts:
    """Lazily quantised (by the oracle) expert weights, from the same bf16
    tensors the GPU path quantised."""

    def __init__(self, cfg: S.MoeConfig):
        import oracle
        self.cfg = cfg
        self.oracle = oracle
        self.cache = {}

    def __call__(self, e: int):
        if e not in self.cache:
            w1, w3, w2 = (host_bits(w) for w in expert_bf16(self.cfg, e))
            self.cache[e] = self.oracle.quantized_expert(w1, w3, w2)
        return self.cache[e]
