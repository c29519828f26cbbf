"""Seeded synthetic inputs for the DeepSeekMoE layer forward.

This module is shared by the CPU oracle (``oracle/``) and the CUDA path
(``fp8_block_scaled_affinity_b200``).  It only draws random numbers and lays
them out; it holds none of the method's arithmetic (no routing, no
quantisation, no expert math).

Workloads follow the shapes of the DeepSeek-V3 MoE layer as summarised on
"DeepSeek-V3 Technical Report" (notes page), section "DeepSeekMoE and
auxiliary-loss-free load balancing": 1 shared + 256 routed experts, 8 routed
experts per token, intermediate size 2048, hidden size 7168 (section
"Pre-training"), token routing limited to M = 4 nodes (read here as expert
groups).

Recipe (all draws in fp32, then rounded to bf16 with round-to-nearest-even):
  * x            ~ N(0, 1)                              bf16 [T, d]
  * router E     ~ N(0, sigma_w)                        bf16 [N_r, d]
  * W1, W3       ~ N(0, sigma_w)                        bf16 [I, d] per expert
  * W2           ~ N(0, sigma_w)                        bf16 [d, I] per expert
  * bias b       ~ U[-beta, beta]                       fp32 [N_r]
  * skewed workload: a Zipf(1.2) prior over experts, passed to routing as an
    fp32 logit offset ln p_i (an input, not part of the method).
  * GEMM-alone workload: A, B ~ N(0, 1), each entry multiplied by 100 with
    probability 0.001 (outliers), then bf16.

Small workloads are drawn on the host with numpy PCG64 so that CPU-only tests
can build them.  The full-size expert weights (11.3 G values) are drawn on
the device with torch's seeded Philox generator, one independent stream per
(expert, matrix), because host generation would take minutes; a test reads
back exactly the tensors the device path consumes.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

__all__ = [
    "MoeConfig", "GemmConfig", "CONFIGS", "GEMM_C2", "get_config",
    "f32_to_bf16_bits", "bf16_bits_to_f32", "host_normal_bf16",
    "host_uniform_f32", "zipf_logit_offset", "make_layer_inputs_host",
    "make_gemm_inputs_host", "device_expert_weights", "host_expert_weights",
]


@dataclasses.dataclass(frozen=True)
class MoeConfig:
    name: str
    T: int            # tokens
    d: int            # hidden size
    n_routed: int     # routed experts N_r
    n_groups: int     # expert groups G (stand-in for nodes)
    topk_groups: int  # M
    topk: int         # K
    inter: int        # expert intermediate size I
    sigma_w: float    # std of router and expert weights
    beta: float       # bias ~ U[-beta, beta]
    gamma: float      # bias update step
    seed: int
    zipf: Optional[float] = None  # Zipf exponent of the logit prior, or None
    batches: int = 1              # successive batches (bias carried over)

    @property
    def rows(self) -> int:
        """Rows of the expert GEMMs: T*K routed pairs plus T shared rows."""
        return self.T * self.topk + self.T


CONFIGS = {
    "tiny": MoeConfig("tiny", T=256, d=512, n_routed=16, n_groups=4,
                      topk_groups=2, topk=4, inter=256, sigma_w=0.02,
                      beta=0.01, gamma=0.001, seed=0),
    "prefill": MoeConfig("prefill", T=4096, d=7168, n_routed=256, n_groups=8,
                         topk_groups=4, topk=8, inter=2048, sigma_w=0.006,
                         beta=0.05, gamma=0.001, seed=2),
    "decode": MoeConfig("decode", T=128, d=7168, n_routed=256, n_groups=8,
                        topk_groups=4, topk=8, inter=2048, sigma_w=0.006,
                        beta=0.05, gamma=0.001, seed=3),
    # profiling case: the prefill layer's per-expert shapes (about 128 rows per
    # expert, d=7168, I=2048) with 16 routed experts, 0.75 GB of FP8 weights
    "prefill_e16": MoeConfig("prefill_e16", T=256, d=7168, n_routed=16, n_groups=8,
                             topk_groups=4, topk=8, inter=2048, sigma_w=0.006,
                             beta=0.05, gamma=0.001, seed=5),
    "skewed": MoeConfig("skewed", T=16384, d=7168, n_routed=256, n_groups=8,
                        topk_groups=4, topk=8, inter=2048, sigma_w=0.006,
                        beta=0.05, gamma=0.001, seed=4, zipf=1.2, batches=8),
}


@dataclasses.dataclass(frozen=True)
class GemmConfig:
    name: str
    m: int
    n: int
    k: int
    outlier_p: float
    outlier_scale: float
    seed: int


GEMM_C2 = GemmConfig("gemm", m=4096, n=2048, k=7168, outlier_p=0.001,
                     outlier_scale=100.0, seed=1)


def get_config(name: str) -> MoeConfig:
    return CONFIGS[name]


# ---------------------------------------------------------------- bf16 bits
def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); return uint16 bits.

    Input construction only: the draws are made in fp32 and stored as bf16.
    NaN is not produced by the generators, so it is not special-cased.
    """
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    r = (b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32)
            << np.uint32(16)).view(np.float32)


def host_normal_bf16(rng: np.random.Generator, shape, sigma: float) -> np.ndarray:
    z = rng.standard_normal(size=shape, dtype=np.float32)
    if sigma != 1.0:
        z = z * np.float32(sigma)
    return f32_to_bf16_bits(z)


def host_uniform_f32(rng: np.random.Generator, shape, beta: float) -> np.ndarray:
    return rng.uniform(-beta, beta, size=shape).astype(np.float32)


def zipf_logit_offset(n_routed: int, s: float) -> np.ndarray:
    """ln p_i for p_i proportional to (i+1)^-s, normalised; fp32 [n_routed].

    Expert index = popularity rank.  This prior skews the token-to-expert
    affinities of the skewed workload; routing receives it as an input.
    """
    i = np.arange(1, n_routed + 1, dtype=np.float64)
    w = i ** (-s)
    return np.log(w / w.sum()).astype(np.float32)


def _rng(*key) -> np.random.Generator:
    return np.random.default_rng(list(key))


def make_layer_inputs_host(cfg: MoeConfig, batch: int = 0) -> dict:
    """Host (numpy) inputs of one batch except the expert weights.

    Returns uint16 bf16 bits for x and the router weight, fp32 for bias and
    the optional logit offset.  Batch j of a multi-batch workload draws x from
    its own stream; router weights and the initial bias do not depend on j.
    """
    x = host_normal_bf16(_rng(cfg.seed, 1, batch), (cfg.T, cfg.d), 1.0)
    router_w = host_normal_bf16(_rng(cfg.seed, 2), (cfg.n_routed, cfg.d), cfg.sigma_w)
    bias = host_uniform_f32(_rng(cfg.seed, 3), (cfg.n_routed,), cfg.beta)
    offset = zipf_logit_offset(cfg.n_routed, cfg.zipf) if cfg.zipf else None
    return {"x": x, "router_w": router_w, "bias": bias, "logit_offset": offset}


def host_expert_weights(cfg: MoeConfig, expert: int):
    """bf16 bits of (W1 [I,d], W3 [I,d], W2 [d,I]) for one expert, drawn on the host.

    Expert index n_routed is the shared expert.  Used for the small workload.
    """
    w1 = host_normal_bf16(_rng(cfg.seed, 10, expert, 1), (cfg.inter, cfg.d), cfg.sigma_w)
    w3 = host_normal_bf16(_rng(cfg.seed, 10, expert, 3), (cfg.inter, cfg.d), cfg.sigma_w)
    w2 = host_normal_bf16(_rng(cfg.seed, 10, expert, 2), (cfg.d, cfg.inter), cfg.sigma_w)
    return w1, w3, w2


def device_expert_weights(cfg: MoeConfig, expert: int, device):
    """bf16 torch tensors (W1, W3, W2) for one expert, drawn on ``device``.

    torch's Philox generator on the device, one seed per (workload, expert,
    matrix).  Deterministic for a given torch version and device type.
    """
    import torch
    out = []
    for mat, shape in ((1, (cfg.inter, cfg.d)), (3, (cfg.inter, cfg.d)),
                       (2, (cfg.d, cfg.inter))):
        g = torch.Generator(device=device)
        g.manual_seed(((cfg.seed * 1009 + expert) * 7 + mat) * 2654435761 % (2 ** 63))
        w = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        out.append((w * cfg.sigma_w).to(torch.bfloat16))
    return tuple(out)


def make_gemm_inputs_host(cfg: GemmConfig = GEMM_C2, m: Optional[int] = None):
    """A [m, k] and B [n, k] (B stored K-major, i.e. the transpose of the
    k x n operand) as bf16 bits, N(0,1) with 0.1% outliers scaled by 100."""
    m = cfg.m if m is None else m
    def draw(key, shape):
        r = _rng(cfg.seed, key)
        z = r.standard_normal(size=shape, dtype=np.float32)
        hit = r.random(size=shape) < cfg.outlier_p
        z = np.where(hit, z * np.float32(cfg.outlier_scale), z)
        return f32_to_bf16_bits(z)
    return draw(1, (m, cfg.k)), draw(2, (cfg.n, cfg.k))
