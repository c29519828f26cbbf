"""Benchmark of the DeepSeekMoE layer forward with FP8 block scaling on B200.

Default workload: the skewed large prefill (T=16384 tokens per batch,
d=7168, 256 routed experts in 8 groups + 1 shared, top-4 groups, K=8,
SwiGLU I=2048, FP8 E4M3 1x128 / 128x128 scales, a Zipf(1.2) prior on the
router logits), eight successive batches cycled, each followed by the
+-gamma bias update.  One step = the whole hot path over one batch: routing
(+ load histogram), 1x128 quantisation of x, permutation, grouped GEMM W13
with SwiGLU + 1x128 quantisation of h, grouped GEMM W2, combine, bias
update.  Expert weights are quantised once before timing (the offline
weight quantisation is timed separately and reported).  Other workloads:
--workload prefill (T=4096), decode (T=128), tiny, gemm (the block-scaled
GEMM alone), route (the router alone), prefill_e16 (a small profiling case).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One process per GPU (torchrun for N > 1).  The path does not shard (one
layer on one GPU): N > 1 runs N independent replicas, each on its own batch
("replicas only", weak scaling); value = all ranks' tokens / max-over-ranks
time.  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE layer tokens/s and expert-GEMM FP8 TFLOPS (% of B200 FP8 dense peak)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_PER_BF16 = 2.0  # nominal dense ratio fp8 : bf16 (4.5 : 2.25 PFLOP/s)
# B200 datasheet figures, reported beside the measured-peak fractions
DATASHEET = {"fp8_tflops": 4500.0, "hbm_gbs": 8000.0}
# Oracle samples (random tokens of the batch): the CPU baseline of the GPU
# arm (one sample, about 10-30 s of host work) and each step of the
# reference arm (so that --steps 20 --warmup 5 ends within a few minutes)
E2E_CALL = 16  # batches per pipelined host-buffer call in the e2e measurement
CPU_SAMPLE_TOKENS = {"tiny": 256, "prefill": 512, "decode": 128, "skewed": 2048,
                     "prefill_e16": 256}
REF_STEP_TOKENS = 64


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", self.gpu_id],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = max(mx, float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------- workload
def algorithmic_counts(cfg, counts_host):
    """Algorithmic FLOPs and bytes of one layer step: the expert GEMMs'
    multiply-adds, the touched experts' FP8 weights, and x in / y out."""
    d, I, K, T = cfg.d, cfg.inter, cfg.topk, cfg.T
    rows = T * K + T
    touched = int((counts_host > 0).sum()) + 1  # + shared expert
    w13_b = 2 * I * d + 4 * (2 * I // 128) * (d // 128)
    w2_b = d * I + 4 * (d // 128) * (I // 128)
    flops_gemm1 = 2.0 * rows * (2 * I) * d
    flops_gemm2 = 2.0 * rows * d * I
    gemm1_bytes = touched * w13_b + rows * (d + 4 * d // 128) + rows * (I + 4 * I // 128)
    gemm2_bytes = touched * w2_b + rows * (I + 4 * I // 128) + rows * d * 4
    layer_bytes = touched * (w13_b + w2_b) + 2 * T * d * 2
    return {"rows": rows, "touched": touched, "flops_gemm1": flops_gemm1,
            "flops_gemm2": flops_gemm2, "gemm1_bytes": gemm1_bytes, "gemm2_bytes": gemm2_bytes,
            "layer_bytes": layer_bytes, "layer_flops": flops_gemm1 + flops_gemm2}


def gemm_source_hash() -> str:
    """Fingerprint of the GEMM kernel's code (comments and blank lines
    ignored), tying a committed DRAM-traffic figure to the code it was
    measured on."""
    h = hashlib.sha256()
    for name in ("gemm.cu", "common.cuh"):
        with open(os.path.join(ROOT, "fp8_block_scaled_affinity_b200", "csrc", name)) as f:
            src = f.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        h.update("\n".join(ln.rstrip() for ln in src.splitlines() if ln.strip()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_tag: str):
    """dram bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", f"{kernel_tag}.txt")
    try:
        text = open(path).read()
    except OSError:
        return None
    m = re.search(r"^source_hash:\s*(\S+)", text, re.M)
    t = re.search(r"^traffic_bytes_per_launch:\s*([0-9.eE+]+)", text, re.M)
    if not m or not t or m.group(1) != gemm_source_hash():
        return None
    return float(t.group(1))


def build_layer(cfg, dev, scales="fp32"):
    import numpy as np
    import torch
    import fp8_block_scaled_affinity_b200 as moe
    import synthetic as S
    inp = S.make_layer_inputs_host(cfg, 0)

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(
            torch.bfloat16).to(dev)

    shape = moe.make_shape(cfg.T, cfg.d, cfg.n_routed, cfg.n_groups, cfg.topk_groups, cfg.topk,
                           cfg.inter, cfg.gamma)
    layer = moe.MoeLayer(shape, bf16(inp["router_w"]), torch.from_numpy(inp["bias"]).to(dev),
                         device=dev, host_io="batches" if scales == "fp32" else False,
                         scales=scales)
    small = cfg.d * cfg.inter <= 512 * 256
    wq_ms = 0.0
    st = torch.cuda.current_stream()
    for e in range(cfg.n_routed + 1):
        if small:
            w = tuple(bf16(m) for m in S.host_expert_weights(cfg, e))
        else:
            w = S.device_expert_weights(cfg, e, dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        layer.set_expert(e, *w)
        b.record(st)
        b.synchronize()
        wq_ms += a.elapsed_time(b)
    x = bf16(inp["x"])
    off = None if inp["logit_offset"] is None else torch.from_numpy(inp["logit_offset"]).to(dev)
    return layer, x, off, inp, wq_ms


def stage_breakdown(layer, x, off, steps):
    """Time each stage of the step on the launching stream with CUDA events
    (the same kernels moe_layer_forward launches, called stage by stage)."""
    import torch
    import fp8_block_scaled_affinity_b200 as moe
    from fp8_block_scaled_affinity_b200 import _lib
    sh = layer.shape
    T, d, I, N, K = sh.T, sh.d, sh.inter, sh.n_routed, sh.topk
    R = T * K + T
    dev = x.device
    xq_p = torch.empty((R, d), dtype=torch.uint8, device=dev)
    xs_p = torch.empty((d // 128, R), dtype=torch.float32, device=dev)
    hq = torch.empty((R, I), dtype=torch.uint8, device=dev)
    hs = torch.empty((I // 128, R), dtype=torch.float32, device=dev)
    o = torch.empty((R, d), dtype=torch.float32, device=dev)
    y = torch.empty_like(x)
    rws = torch.empty((moe.moe_route_workspace_size(sh),), dtype=torch.uint8, device=dev)
    pws = torch.empty((moe.moe_permute_workspace_size(sh),), dtype=torch.uint8, device=dev)
    st = torch.cuda.current_stream()
    names = ["route", "quant_permute", "gemm1_swiglu", "gemm2", "combine", "update_bias"]
    mx = getattr(layer, "scales", "fp32") == "ue8m0"
    if mx:  # power-of-two option: UE8M0 scale bytes, block-scaled GEMMs
        xs_p = torch.empty((d // 128, R), dtype=torch.uint8, device=dev)
        hs = torch.empty((I // 128, R), dtype=torch.uint8, device=dev)
    permute = moe.moe_quant_permute_ue8m0 if mx else moe.moe_quant_permute
    gemm = moe.moe_grouped_gemm_mxfp8 if mx else moe.moe_grouped_gemm_fp8
    calls = [
        lambda: moe.moe_route(sh, x, layer.router_w, layer.bias, off, layer.topk_idx,
                              layer.topk_gate, layer.expert_counts, rws),
        lambda: permute(sh, x, layer.topk_idx, layer.expert_counts, xq_p, xs_p,
                        layer.expert_offsets, layer.row_of_pair, pws),
        lambda: gemm(N + 1, layer.expert_offsets, R, xq_p, xs_p, d, layer.w13, layer.w13_scales,
                     2 * I, _lib.MOE_EPI_SWIGLU_QUANT, hq, hs, layer.dev_status),
        lambda: gemm(N + 1, layer.expert_offsets, R, hq, hs, I, layer.w2, layer.w2_scales, d,
                     _lib.MOE_EPI_F32, o, None, layer.dev_status),
        lambda: moe.moe_combine(sh, o, layer.expert_offsets, layer.row_of_pair,
                                layer.topk_gate, y),
        lambda: moe.moe_update_bias(sh, layer.expert_counts, layer.bias),
    ]
    tot = {n: 0.0 for n in names}
    for it in range(steps + 2):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)]
        ev[0].record(st)
        for i, c in enumerate(calls):
            c()
            ev[i + 1].record(st)
        ev[-1].synchronize()
        if it >= 2:
            for i, n in enumerate(names):
                tot[n] += ev[i].elapsed_time(ev[i + 1])
    return {n: tot[n] / steps for n in names}


# ------------------------------------------------------------ CPU oracle
_ORACLE_WEIGHTS = {}  # workload -> expert -> oracle-quantised weights (reused across samples)


def oracle_sample_time(cfg, inp, dev, n_tokens, seed=0):
    """The oracle (as it stands) on a bounded sample: n_tokens tokens through
    routing, quantisation, the experts they touch and the combine.  Expert
    weights are quantised by the oracle beforehand (untimed, like the GPU
    path's offline weight quantisation).  Returns (seconds, tokens, cores)."""
    import numpy as np
    import torch
    import oracle
    import synthetic as S
    rng = np.random.default_rng(seed)
    toks = np.sort(rng.choice(cfg.T, n_tokens, replace=False))
    x = inp["x"][toks]
    r = oracle.route(x, inp["router_w"], inp["bias"], cfg.n_groups, cfg.topk_groups, cfg.topk,
                     logit_offset=inp["logit_offset"])
    need = sorted(set(r["topk_idx"].ravel().tolist()) | {cfg.n_routed})
    small = cfg.d * cfg.inter <= 512 * 256
    W = _ORACLE_WEIGHTS.setdefault(cfg.name, {})
    for e in need:
        if e in W:
            continue
        if small:
            w = S.host_expert_weights(cfg, e)
        else:
            w = tuple(t.cpu().view(torch.int16).numpy().view(np.uint16)
                      for t in S.device_expert_weights(cfg, e, dev))
        W[e] = oracle.quantized_expert(*w)
    t0 = time.perf_counter()
    oracle.layer_forward(x, inp["router_w"], inp["bias"], cfg.n_groups, cfg.topk_groups,
                         cfg.topk, W.__getitem__, logit_offset=inp["logit_offset"])
    dt = time.perf_counter() - t0
    return dt, n_tokens, os.cpu_count() or 1


# ------------------------------------------------------ memory-bound passes
def memory_passes(cfg, brk, alg, hbm_peak):
    """Algorithmic bytes / event time of the HBM-bound passes of one step."""
    T, d, K = cfg.T, cfg.d, cfg.topk
    nkb = d // 128
    rows = T * K + T
    passes = {
        # bf16 row read once, E4M3 row + 1x128 scales written to K+1 rows
        "quant_permute": (brk["quant_permute"], T * d * 2 + rows * (d + 4 * nkb)),
        # fp32 expert rows read (K routed + shared) and gates, bf16 y written
        "combine": (brk["combine"], rows * d * 4 + T * K * 8 + T * d * 2),
    }
    out = {}
    for name, (ms, nbytes) in passes.items():
        gbs = nbytes / (ms / 1e3) / 1e9
        out[name] = {"ms": ms, "bytes": nbytes, "gbs": gbs, "frac_of_hbm": gbs / hbm_peak,
                     "frac_of_datasheet": gbs / DATASHEET["hbm_gbs"]}
    return out


def weight_quant_pass(dev, hbm_peak, rows=32768, cols=7168, reps=5):
    """fp8_quant_w_128x128 timed alone on one [rows, cols] bf16 matrix (the
    stacked W1/W3 of 8 experts; 0.7 GB moved, above L2)."""
    import torch
    import fp8_block_scaled_affinity_b200 as moe
    g = torch.Generator(device=dev)
    g.manual_seed(7)
    w = (torch.randn((rows, cols), generator=g, device=dev) * 0.006).to(torch.bfloat16)
    q = torch.empty((rows, cols), dtype=torch.uint8, device=dev)
    sc = torch.empty((rows // 128, cols // 128), dtype=torch.float32, device=dev)
    st = torch.cuda.current_stream()
    for _ in range(2):
        moe.fp8_quant_w_128x128(w, q, sc)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ev[0].record(st)
    for _ in range(reps):
        moe.fp8_quant_w_128x128(w, q, sc)
    ev[1].record(st)
    ev[1].synchronize()
    ms = ev[0].elapsed_time(ev[1]) / reps
    nbytes = rows * cols * 3 + 4 * (rows // 128) * (cols // 128)
    gbs = nbytes / (ms / 1e3) / 1e9
    del w, q, sc
    return {"ms": ms, "shape": [rows, cols], "bytes": nbytes, "gbs": gbs,
            "frac_of_hbm": gbs / hbm_peak, "frac_of_datasheet": gbs / DATASHEET["hbm_gbs"]}


# ------------------------------------------------------------ router alone
INT8_PLANE_PRODUCTS = 16  # 4 x 4 digit planes multiplied by the router's tensor-core kernel


def run_route(args, world, rank, local):
    """moe_route alone on the prefill batch (T=4096, d=7168, 256 experts):
    logits, sigmoid, group-limited top-K, gates and histogram.  The logits
    come from 16 int8 digit-plane products of T*N_r*d multiply-adds each on
    the tensor cores; the roofline line reports their rate over the whole
    call (all six router kernels) against the dense 8-bit tensor peak."""
    import numpy as np
    import torch
    import fp8_block_scaled_affinity_b200 as moe
    import synthetic as S
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    cfg = S.CONFIGS["prefill"]
    inp = S.make_layer_inputs_host(cfg, 0)

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(
            torch.bfloat16).to(dev)

    x, rw = bf16(inp["x"]), bf16(inp["router_w"])
    bias = torch.from_numpy(inp["bias"]).to(dev)
    shape = moe.make_shape(cfg.T, cfg.d, cfg.n_routed, cfg.n_groups, cfg.topk_groups, cfg.topk,
                           cfg.inter, cfg.gamma)
    idx = torch.empty((cfg.T, cfg.topk), dtype=torch.int32, device=dev)
    gate = torch.empty((cfg.T, cfg.topk), dtype=torch.float32, device=dev)
    counts = torch.empty((cfg.n_routed,), dtype=torch.int32, device=dev)
    ws = torch.empty((moe.moe_route_workspace_size(shape),), dtype=torch.uint8, device=dev)
    status = torch.zeros((1,), dtype=torch.int32, device=dev)
    flush = torch.empty((256 << 20,), dtype=torch.uint8, device=dev)
    st = torch.cuda.current_stream()

    def route(xx=x):
        moe.moe_route(shape, xx, rw, bias, None, idx, gate, counts, ws, status)

    for _ in range(args.warmup):
        flush.fill_(1)
        route()
    torch.cuda.synchronize()
    barrier(world)
    props = torch.cuda.get_device_properties(dev)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local)
    clocks = ClockSampler(gpu_id)
    clocks.start()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for e0, e1 in evs:
        flush.fill_(1)
        e0.record(st)
        route()
        e1.record(st)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier(world)
    ms = max_over_ranks(sum(e0.elapsed_time(e1) for e0, e1 in evs), world)
    fma = float(cfg.T) * cfg.n_routed * cfg.d
    peaks, peak_src = load_peaks()
    tops = 2.0 * INT8_PLANE_PRODUCTS * fma * args.steps * world / (ms / 1e3) / 1e12
    peak = float(peaks["bf16_tflops"]) * FP8_PER_BF16
    x_h = x.cpu().pin_memory()
    x_d = torch.empty_like(x)
    idx_h = torch.empty((cfg.T, cfg.topk), dtype=torch.int32).pin_memory()
    gate_h = torch.empty((cfg.T, cfg.topk), dtype=torch.float32).pin_memory()
    e2e_ms = 0.0
    for it in range(args.warmup + args.steps):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        x_d.copy_(x_h, non_blocking=True)
        route(x_d)
        idx_h.copy_(idx, non_blocking=True)
        gate_h.copy_(gate, non_blocking=True)
        e1.record(st)
        e1.synchronize()
        if it >= args.warmup:
            e2e_ms += e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(e2e_ms, world)
    tok = cfg.T * args.steps * world
    line = {
        "metric": METRIC, "value": tok / (ms / 1e3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8/f64", "data": "synthetic",
        "config": {"workload": "moe_route_prefill", "T": cfg.T, "d": cfg.d,
                   "n_routed": cfg.n_routed, "n_groups": cfg.n_groups,
                   "topk_groups": cfg.topk_groups, "topk": cfg.topk,
                   "parallelism": f"replicas x{world}",
                   "l2": "256 MB buffer written between timed launches"},
        "roofline": {"bound": "tensor",
                     "kernel": "moe_route (int8 digit-plane logits on tcgen05 + certification)",
                     "achieved": tops / world, "peak": peak, "unit": "TOP/s",
                     "frac": tops / world / peak,
                     "peak_source": f"{peak_src} bf16 burst x {FP8_PER_BF16:g} (8-bit:bf16 nominal)",
                     "traffic": None,
                     "algorithmic_int8_macs_per_launch": INT8_PLANE_PRODUCTS * fma,
                     "definition_fma_per_launch": fma},
        "e2e": {"value": tok / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": x.numel() * 2,
                "d2h_bytes_per_step": idx.numel() * 4 + gate.numel() * 4},
        "gpu_launches": 8 * args.steps,  # the router's kernels
        "clocks": clk,
        "device_status": int(status.item()),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_permute(args, world, rank, local):
    """The 1x128 activation quantisation fused with the permutation copy
    (moe_quant_permute) alone, on the prefill batch (T=4096, d=7168, K=8):
    x read once in bf16, codes and kb-major scales written to the K + 1
    destination rows.  Routing runs once beforehand, untimed; a 256 MB buffer
    is written between timed launches (x is smaller than L2)."""
    import numpy as np
    import torch
    import fp8_block_scaled_affinity_b200 as moe
    import synthetic as S
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    cfg = S.CONFIGS["prefill"]
    inp = S.make_layer_inputs_host(cfg, 0)

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(
            torch.bfloat16).to(dev)

    x, rw = bf16(inp["x"]), bf16(inp["router_w"])
    bias = torch.from_numpy(inp["bias"]).to(dev)
    T, d, K, N = cfg.T, cfg.d, cfg.topk, cfg.n_routed
    R = T * K + T
    shape = moe.make_shape(T, d, N, cfg.n_groups, cfg.topk_groups, K, cfg.inter, cfg.gamma)
    idx = torch.empty((T, K), dtype=torch.int32, device=dev)
    gate = torch.empty((T, K), dtype=torch.float32, device=dev)
    counts = torch.empty((N,), dtype=torch.int32, device=dev)
    rws = torch.empty((moe.moe_route_workspace_size(shape),), dtype=torch.uint8, device=dev)
    status = torch.zeros((1,), dtype=torch.int32, device=dev)
    moe.moe_route(shape, x, rw, bias, None, idx, gate, counts, rws, status)
    xq = torch.empty((R, d), dtype=torch.uint8, device=dev)
    xs = torch.empty((d // 128, R), dtype=torch.float32, device=dev)
    off = torch.empty((N + 2,), dtype=torch.int32, device=dev)
    rop = torch.empty((T, K), dtype=torch.int32, device=dev)
    pws = torch.empty((moe.moe_permute_workspace_size(shape),), dtype=torch.uint8, device=dev)
    flush = torch.empty((256 << 20,), dtype=torch.uint8, device=dev)
    st = torch.cuda.current_stream()

    def step():
        moe.moe_quant_permute(shape, x, idx, counts, xq, xs, off, rop, pws, status)

    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()
    barrier(world)
    props = torch.cuda.get_device_properties(dev)
    clocks = ClockSampler(f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local))
    clocks.start()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for e0, e1 in evs:
        flush.fill_(1)
        e0.record(st)
        step()
        e1.record(st)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier(world)
    ms = max_over_ranks(sum(e0.elapsed_time(e1) for e0, e1 in evs), world)
    peaks, peak_src = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    nbytes = T * d * 2 + R * (d + 4 * (d // 128))  # x in; codes + scales out
    gbs = nbytes * args.steps / (ms / 1e3) / 1e9
    tok = T * args.steps * world
    line = {
        "metric": METRIC, "value": tok / (ms / 1e3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16->fp8e4m3", "data": "synthetic",
        "config": {"workload": "moe_quant_permute_prefill", "T": T, "d": d, "n_routed": N,
                   "topk": K, "parallelism": f"replicas x{world}",
                   "l2": "256 MB buffer written between timed launches"},
        "roofline": {"bound": "hbm", "kernel": "quant_copy_rows_kernel (+ permutation ranks)",
                     "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                     "peak_source": peak_src, "traffic": None,
                     "algorithmic_bytes_per_launch": nbytes,
                     "frac_of_datasheet": gbs / DATASHEET["hbm_gbs"]},
        "e2e": None,
        "gpu_launches": 4 * args.steps,
        "clocks": clk,
        "device_status": int(status.item()),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_ep(args, world, rank, local):
    """Expert-parallel layer stages, P = 8 ranks emulated on one GPU: each
    rank owns 32 of the prefill layer's 256 routed experts (plus the shared
    one) and routes its own 2,048 tokens (16,384 in all); every rank's
    stages run through the library and each all-to-all is a device copy
    that hands rank p's rows for rank q to rank q.  All ranks' stages run
    one after another on one stream, so the value is the serialised
    throughput of the EP kernels, not a multi-GPU figure; the per-stage
    times and the EP kernels' GB/s are the point."""
    import numpy as np
    import torch
    import fp8_block_scaled_affinity_b200 as moe
    from fp8_block_scaled_affinity_b200.ep import EpMoeLayer
    import synthetic as S
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    cfg = S.CONFIGS["prefill"]
    P, T = 8, 2048
    inp = S.make_layer_inputs_host(cfg, 0)

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(
            torch.bfloat16).to(dev)

    shape = moe.make_shape(T, cfg.d, cfg.n_routed, cfg.n_groups, cfg.topk_groups, cfg.topk,
                           cfg.inter, cfg.gamma)
    rw, bias = bf16(inp["router_w"]), torch.from_numpy(inp["bias"]).to(dev)
    layers = [EpMoeLayer(shape, q, P, rw, bias.clone(), device=dev) for q in range(P)]
    for e in range(cfg.n_routed + 1):
        w = S.device_expert_weights(cfg, e, dev)
        for l in layers:
            l.set_expert(e, *w)
    xs = [bf16(S.make_layer_inputs_host(cfg, 1 + q)["x"][:T]) for q in range(P)]
    d = cfg.d

    def step(marks=None):
        sends = [l.route_and_pack(x, marks=marks) for l, x in zip(layers, xs)]
        offs = [np.concatenate([[0], np.cumsum(c)]) for _, c in sends]
        recv, src = [], []
        for q in range(P):  # the dispatch all-to-all as device copies
            recv.append(torch.cat([sends[p][0][offs[p][q]:offs[p][q + 1]] for p in range(P)]))
            src.append(np.concatenate([[0], np.cumsum([sends[p][1][q] for p in range(P)])]))
        backs = [layers[q].experts(recv[q], int(src[q][-1]), marks=marks) for q in range(P)]
        ys = []
        for p in range(P):  # the combine all-to-all as device copies
            back = torch.cat([backs[q][src[q][p]:src[q][p + 1]] for q in range(P)])
            ys.append(layers[p].shared_and_combine(xs[p], back, marks=marks))
        return sends, recv

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    props = torch.cuda.get_device_properties(dev)
    clocks = ClockSampler(f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local))
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(args.steps):
        sends, recv = step()
    e1.record(st)
    e1.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1)
    # per-stage times, all ranks summed (events between the library calls)
    tot = {}
    for it in range(args.steps):
        marks = []
        step(marks)
        torch.cuda.synchronize()
        prev = None
        for name, ev in marks:
            if name != "start" and prev is not None:
                tot[name] = tot.get(name, 0.0) + prev.elapsed_time(ev)
            prev = ev
    brk = {n: v / args.steps for n, v in tot.items()}
    n_send = sum(sum(c) for _, c in sends)
    rb = layers[0].row_bytes
    K, nkb = cfg.topk, d // 128
    local_rows = sum(int(l.counts.sum().item()) for l in layers)  # routed pairs, all ranks
    peaks, peak_src = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    ep_bytes = {
        # x read (bf16) + the rows written
        "pack": P * T * d * 2 + n_send * rb,
        # rows read + the local FP8 rows and kb-major scales written
        "local_permute": n_send * rb + local_rows * (d + 4 * nkb),
        # fp32 expert rows read + one fp32 partial row per received row written
        "partial_combine": local_rows * d * 4 + n_send * d * 4,
        # shared output + partial rows read (fp32), y written (bf16)
        "final_combine": P * T * d * 4 + n_send * d * 4 + P * T * d * 2,
    }
    passes = {n: {"ms": brk[n], "bytes": b, "gbs": b / (brk[n] / 1e3) / 1e9,
                  "frac_of_hbm": b / (brk[n] / 1e3) / 1e9 / hbm}
              for n, b in ep_bytes.items()}
    top = max(ep_bytes, key=lambda n: brk[n])
    tok = P * T * args.steps
    line = {
        "metric": "ep_emulated_tokens_per_s", "value": tok / (ms / 1e3), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp8e4m3/f32", "data": "synthetic",
        "config": {"workload": "moe_ep_prefill_8_ranks_on_one_gpu", "ranks": P,
                   "tokens_per_rank": T, "d": d, "n_routed": cfg.n_routed,
                   "experts_per_rank": cfg.n_routed // P, "topk": K, "inter": cfg.inter,
                   "exchange": "device copies standing in for the all-to-alls",
                   "l2": "inputs larger than L2 (11.6 GB of FP8 weights over the ranks)"},
        "roofline": {"bound": "hbm", "kernel": f"EP {top}", "achieved": passes[top]["gbs"],
                     "peak": hbm, "unit": "GB/s", "frac": passes[top]["frac_of_hbm"],
                     "peak_source": peak_src, "traffic": None,
                     "algorithmic_bytes_per_launch": ep_bytes[top] / P,
                     "frac_of_datasheet": passes[top]["gbs"] / DATASHEET["hbm_gbs"]},
        "ep_passes": passes,
        "breakdown_ms": brk,
        "dispatch_rows": n_send, "row_bytes": rb,
        "rows_per_token": n_send / (P * T),
        "e2e": None,
        "gpu_launches": None,
        "clocks": clk,
        "device_status": int(sum(int(l.dev_status.item()) for l in layers)),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_redundant(args, world, rank, local):
    """Redundant experts on the skewed batch (T=16384): after one forward
    pass, the planner gives 32 extra copies to the hottest experts and the
    two expert GEMMs run over the copies' groups (each copy a group of the
    indexed grouped GEMM sharing its expert's weights; the output rows are
    bit-identical).  Both GEMMs are timed with and without the copies."""
    import numpy as np
    import torch
    import fp8_block_scaled_affinity_b200 as moe
    import synthetic as S
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    cfg = S.CONFIGS["skewed"]
    layer, x, off, inp, _ = build_layer(cfg, dev)
    y = layer.forward(x, logit_offset=off)
    torch.cuda.synchronize()
    sh = layer.shape
    T, d, I, N, K = cfg.T, cfg.d, cfg.inter, cfg.n_routed, cfg.topk
    R = T * K + T
    n_extra = 32
    counts = layer.expert_counts.cpu().numpy()
    rep, slots = moe.moe_plan_redundant_experts(counts, n_extra)
    first = np.concatenate([[0], np.cumsum(rep)[:-1]]).astype(np.int32)
    G = N + n_extra + 1
    so = torch.empty(G + 1, dtype=torch.int32, device=dev)
    sw = torch.empty(G, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    todev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    moe.moe_split_groups(sh, layer.expert_offsets, todev(rep), todev(slots), todev(first), n_extra,
                         so, sw, status)
    xq = torch.empty((R, d), dtype=torch.uint8, device=dev)
    xs = torch.empty((d // 128, R), dtype=torch.float32, device=dev)
    hq = torch.empty((R, I), dtype=torch.uint8, device=dev)
    hs = torch.empty((I // 128, R), dtype=torch.float32, device=dev)
    o = torch.empty((R, d), dtype=torch.float32, device=dev)
    pws = torch.empty((moe.moe_permute_workspace_size(sh),), dtype=torch.uint8, device=dev)
    moe.moe_quant_permute(sh, x, layer.topk_idx, layer.expert_counts, xq, xs,
                          layer.expert_offsets, layer.row_of_pair, pws)
    st = torch.cuda.current_stream()

    def gemms(copies):
        if copies:
            moe.moe_grouped_gemm_fp8_indexed(G, so, sw, N + 1, R, xq, xs, d, layer.w13,
                                             layer.w13_scales, 2 * I, moe.MOE_EPI_SWIGLU_QUANT,
                                             hq, hs, status)
            moe.moe_grouped_gemm_fp8_indexed(G, so, sw, N + 1, R, hq, hs, I, layer.w2,
                                             layer.w2_scales, d, moe.MOE_EPI_F32, o, None,
                                             status)
        else:
            moe.moe_grouped_gemm_fp8(N + 1, layer.expert_offsets, R, xq, xs, d, layer.w13,
                                     layer.w13_scales, 2 * I, moe.MOE_EPI_SWIGLU_QUANT, hq, hs,
                                     status)
            moe.moe_grouped_gemm_fp8(N + 1, layer.expert_offsets, R, hq, hs, I, layer.w2,
                                     layer.w2_scales, d, moe.MOE_EPI_F32, o, None, status)

    res = {}
    for copies in (False, True, False, True):
        for _ in range(args.warmup):
            gemms(copies)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        for _ in range(args.steps):
            gemms(copies)
        e1.record(st)
        e1.synchronize()
        res.setdefault(copies, []).append(e0.elapsed_time(e1) / args.steps)
    ms_plain, ms_copies = min(res[False]), min(res[True])
    flops = 2.0 * R * d * 3 * I
    peaks, peak_src = load_peaks()
    fp8_peak = float(peaks["bf16_tflops"]) * FP8_PER_BF16
    tf = flops / (ms_copies / 1e3) / 1e12
    sizes = np.diff(so.cpu().numpy())[:-1]
    line = {
        "metric": "expert_gemm_tflops", "value": tf, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_copies,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8e4m3/f32", "data": "synthetic",
        "config": {"workload": "redundant_experts_skewed", "T": T, "n_extra": n_extra,
                   "groups": G, "largest_group_rows": int(sizes.max()),
                   "largest_expert_rows": int(counts.max()),
                   "l2": "inputs larger than L2 (11.3 GB of FP8 weights)"},
        "roofline": {"bound": "tensor", "kernel": "grouped_gemm (W13 + W2) over the copies",
                     "achieved": tf, "peak": fp8_peak, "unit": "TFLOP/s", "frac": tf / fp8_peak,
                     "peak_source": f"{peak_src} bf16 burst x {FP8_PER_BF16:g}", "traffic": None,
                     "frac_of_datasheet": tf / DATASHEET["fp8_tflops"]},
        "without_copies": {"ms": ms_plain, "tflops": flops / (ms_plain / 1e3) / 1e12},
        "with_copies": {"ms": ms_copies, "tflops": tf},
        "e2e": None,
        "gpu_launches": 2 * args.steps,
        "device_status": int(status.item()),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------- GEMM-alone workload
def run_gemm(args, world, rank, local):
    """The FP8 block-scaled GEMM alone: A [4096, 7168] (1x128 scales) times B
    [7168, 2048] (128x128 scales, stored K-major as [2048, 7168]), bf16 out.
    One step = one moe_grouped_gemm_fp8 launch (one group); a 256 MB buffer
    is written between steps (outside the timed events) so each launch reads
    its operands from HBM."""
    import numpy as np
    import torch
    import fp8_block_scaled_affinity_b200 as moe
    import synthetic as S
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    cfg = S.GEMM_C2
    peaks, peak_src = load_peaks()
    a_bits, b_bits = S.make_gemm_inputs_host(cfg)

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(
            torch.bfloat16).to(dev)

    a, b = bf16(a_bits), bf16(b_bits)
    mx = args.scales == "ue8m0"
    sdt = torch.uint8 if mx else torch.float32
    aq = torch.empty((cfg.m, cfg.k), dtype=torch.uint8, device=dev)
    as_ = torch.empty((cfg.k // 128, cfg.m), dtype=sdt, device=dev)
    bq = torch.empty((cfg.n, cfg.k), dtype=torch.uint8, device=dev)
    bs = torch.empty((cfg.n // 128, cfg.k // 128), dtype=sdt, device=dev)
    if mx:  # power-of-two option: UE8M0 scale bytes, block-scaled GEMM
        moe.fp8_quant_act_1x128_ue8m0(a, aq, as_, sf_kb_major=True)
        moe.fp8_quant_w_128x128_ue8m0(b, bq, bs)
    else:
        moe.fp8_quant_act_1x128(a, aq, as_, scales_kb_major=True)
        moe.fp8_quant_w_128x128(b, bq, bs)
    gemm_fn = moe.moe_grouped_gemm_mxfp8 if mx else moe.moe_grouped_gemm_fp8
    off = torch.tensor([0, cfg.m], dtype=torch.int32, device=dev)
    out = torch.empty((cfg.m, cfg.n), dtype=torch.bfloat16, device=dev)
    status = torch.zeros((1,), dtype=torch.int32, device=dev)
    flush = torch.empty((256 << 20,), dtype=torch.uint8, device=dev)
    st = torch.cuda.current_stream()

    form = moe.moe_grouped_gemm_form(1, cfg.m, cfg.n, moe.MOE_EPI_BF16)

    def gemm(a_codes=aq, a_scales=as_, c=out):
        gemm_fn(1, off, cfg.m, a_codes, a_scales, cfg.k, bq, bs, cfg.n,
                                 moe.MOE_EPI_BF16, c, None, status)

    for _ in range(args.warmup):
        flush.fill_(1)
        gemm()
    torch.cuda.synchronize()
    barrier(world)
    props = torch.cuda.get_device_properties(dev)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local)
    clocks = ClockSampler(gpu_id)
    clocks.start()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for e0, e1 in evs:
        flush.fill_(1)
        e0.record(st)
        gemm()
        e1.record(st)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier(world)
    ms = max_over_ranks(sum(e0.elapsed_time(e1) for e0, e1 in evs), world)
    flops = 2.0 * cfg.m * cfg.n * cfg.k
    tflops = flops * args.steps * world / (ms / 1e3) / 1e12
    fp8_peak = float(peaks["bf16_tflops"]) * FP8_PER_BF16

    # end to end: A's codes and scales from pinned host memory, C back to it
    aq_h, as_h = aq.cpu().pin_memory(), as_.cpu().pin_memory()
    c_h = torch.empty((cfg.m, cfg.n), dtype=torch.bfloat16).pin_memory()
    aq_d, as_d = torch.empty_like(aq), torch.empty_like(as_)
    e2e_ms = 0.0
    for it in range(args.warmup + args.steps):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        aq_d.copy_(aq_h, non_blocking=True)
        as_d.copy_(as_h, non_blocking=True)
        gemm(aq_d, as_d, out)
        c_h.copy_(out, non_blocking=True)
        e1.record(st)
        e1.synchronize()
        if it >= args.warmup:
            e2e_ms += e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(e2e_ms, world)
    line = {
        "metric": METRIC, "value": tflops, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8e4m3/f32", "data": "synthetic",
        "config": {"workload": "fp8_blockscaled_gemm", "scales": args.scales,
                   "m": cfg.m, "n": cfg.n, "k": cfg.k,
                   "out": "bf16", "parallelism": f"replicas x{world}",
                   "l2": "256 MB buffer written between timed launches"},
        "roofline": {"bound": "tensor",
                     "kernel": ("mx_gemm_kernel<0> (block-scaled, UE8M0 scales; one group, "
                                "bf16 out)" if mx else
                                f"grouped_gemm_kernel<{int(form == 2)}, 0, 1> "
                                f"({'CTA pairs' if form == 2 else 'single CTAs'}; one group, "
                                "bf16 out)"),
                     "achieved": tflops / world, "peak": fp8_peak, "unit": "TFLOP/s",
                     "frac": tflops / world / fp8_peak,
                     "frac_of_datasheet": tflops / world / DATASHEET["fp8_tflops"],
                     "datasheet_peak": DATASHEET["fp8_tflops"],
                     "peak_source": f"{peak_src} bf16 burst x {FP8_PER_BF16:g} (nominal fp8:bf16)",
                     "traffic": profiled_traffic("gemm_ue8m0_4096x7168x2048" if mx else
                                                 "gemm_blockscaled_4096x7168x2048"),
                     "algorithmic_flops_per_launch": flops, "launch_ms": ms / args.steps},
        "e2e": {"value": flops * args.steps * world / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": aq.numel() + as_.numel() * 4,
                "d2h_bytes_per_step": out.numel() * 2},
        "gpu_launches": args.steps,
        "clocks": clk,
        "device_status": int(status.item()),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        n_rows = 16
        qa, sa = oracle.quant_act_1x128(a_bits[:n_rows])
        qb, sb = oracle.quant_w_128x128(b_bits)
        t0 = time.perf_counter()
        oracle.gemm_blockscaled(qa, sa, qb, sb)
        dt = time.perf_counter() - t0
        line["cpu_baseline"] = {
            "value": 2.0 * n_rows * cfg.n * cfg.k / dt / 1e12, "unit": "TFLOP/s",
            "cores": os.cpu_count() or 1, "kind": "oracle",
            "sample": f"{n_rows} rows of A times all of B (operands pre-quantised by the oracle)"}
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------- main
def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return world, rank, local


def max_over_ranks(value: float, world: int) -> float:
    """Max of a host float over all ranks (identity for one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def run_reference(args, world, rank):
    """The oracle timed on the host cores: each step is a bounded sample of
    the workload (REF_STEP_TOKENS random tokens)."""
    import numpy as np
    import torch
    import synthetic as S
    if rank != 0:
        return
    if args.workload == "gemm":
        return run_reference_gemm(args)
    if args.workload == "route":
        return run_reference_route(args)
    cfg = S.CONFIGS[args.workload]
    dev = torch.device("cuda:0") if torch.cuda.is_available() else torch.device("cpu")
    inp = S.make_layer_inputs_host(cfg, 0)
    times = []
    n_tok = min(REF_STEP_TOKENS, cfg.T)
    for i in range(args.warmup + args.steps):
        dt, n, cores = oracle_sample_time(cfg, inp, dev, n_tok, seed=i)
        if i >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = args.steps * n_tok / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"moe_layer_{cfg.name}", "T": cfg.T, "d": cfg.d,
                   "n_routed": cfg.n_routed, "n_shared": 1, "n_groups": cfg.n_groups,
                   "topk_groups": cfg.topk_groups, "topk": cfg.topk, "inter": cfg.inter,
                   "sample_tokens_per_step": n_tok},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": os.cpu_count() or 1,
                         "kind": "oracle",
                         "sample": f"{n_tok} random tokens per step of the "
                                   f"{cfg.name} batch (routing, quantisation, touched experts,"
                                   " combine)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_reference_route(args, n_tok=64):
    """The oracle's routing on n_tok tokens of the prefill batch per step."""
    import oracle
    import synthetic as S
    cfg = S.CONFIGS["prefill"]
    inp = S.make_layer_inputs_host(cfg, 0)
    times = []
    for i in range(args.warmup + args.steps):
        t0_ = (i * n_tok) % cfg.T
        xs = inp["x"][t0_:t0_ + n_tok]
        t0 = time.perf_counter()
        oracle.route(xs, inp["router_w"], inp["bias"], cfg.n_groups, cfg.topk_groups, cfg.topk)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    total = sum(times)
    value = n_tok * args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "moe_route_prefill", "T": cfg.T, "d": cfg.d,
                   "n_routed": cfg.n_routed, "n_groups": cfg.n_groups,
                   "topk_groups": cfg.topk_groups, "topk": cfg.topk,
                   "sample_tokens_per_step": n_tok},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": os.cpu_count() or 1,
                         "kind": "oracle", "sample": f"{n_tok} tokens per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_reference_gemm(args, n_rows=16):
    """The oracle's block-scaled GEMM on n_rows rows of A per step (operands
    quantised by the oracle beforehand, untimed)."""
    import oracle
    import synthetic as S
    cfg = S.GEMM_C2
    a_bits, b_bits = S.make_gemm_inputs_host(cfg)
    qb, sb = oracle.quant_w_128x128(b_bits)
    times = []
    for i in range(args.warmup + args.steps):
        r0 = (i * n_rows) % cfg.m
        qa, sa = oracle.quant_act_1x128(a_bits[r0:r0 + n_rows])
        t0 = time.perf_counter()
        oracle.gemm_blockscaled(qa, sa, qb, sb)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    total = sum(times)
    value = 2.0 * n_rows * cfg.n * cfg.k * args.steps / total / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "fp8_blockscaled_gemm", "m": cfg.m, "n": cfg.n, "k": cfg.k,
                   "out": "bf16", "sample_rows_per_step": n_rows},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": os.cpu_count() or 1,
                         "kind": "oracle",
                         "sample": f"{n_rows} rows of A per step times all of B"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, world, rank, local):
    import numpy as np
    import torch
    import fp8_block_scaled_affinity_b200 as moe
    import synthetic as S

    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    cfg = S.CONFIGS[args.workload]
    peaks, peak_src = load_peaks()
    layer, x, off, inp, wq_ms = build_layer(cfg, dev, args.scales)
    st = torch.cuda.current_stream()
    y = torch.empty_like(x)
    bias0 = layer.bias.clone()
    # successive batches (the skewed workload has 8; step i routes batch
    # i mod 8 with the bias left by step i-1)
    batches = [x] + [torch.from_numpy(np.ascontiguousarray(
        S.make_layer_inputs_host(cfg, j)["x"]).view(np.int16)).view(torch.bfloat16).to(dev)
        for j in range(1, cfg.batches)]
    nb = len(batches)

    # ---- warm-up, then K timed steps of the whole layer (inputs in HBM)
    for i in range(args.warmup):
        layer.forward(batches[i % nb], y, update_bias=True, logit_offset=off)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(dev)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local)
    clocks = ClockSampler(gpu_id)
    clocks.start()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(st)
    for i in range(args.steps):
        layer.forward(batches[i % nb], y, update_bias=True, logit_offset=off)
    ev1.record(st)
    ev1.synchronize()
    clk = clocks.stop()
    barrier(world)
    ms_local = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms_local, world)
    status = layer.status()
    counts = layer.expert_counts.cpu().numpy()
    tokens_total = cfg.T * args.steps * world
    value = tokens_total / (ms / 1e3)

    # ---- end to end through the host-buffer entry points (pinned memory):
    # the batches call overlaps each batch's copies with its neighbours'
    # compute; one forward_host call per step (copies in line) is reported
    # beside it
    # the steps' batches (batch i mod 8) in pinned host memory, in order, at
    # most E2E_CALL of them per call (bounded pinned memory: 3.8 GB each way)
    per_call = min(args.steps, E2E_CALL)
    x_hosts = torch.stack([batches[i % nb].cpu() for i in range(per_call)]).pin_memory()
    y_hosts = torch.empty_like(x_hosts).pin_memory()

    def e2e_steps(pipelined):
        done = 0
        while done < args.steps:
            n = min(per_call, args.steps - done)
            if pipelined:  # the copies overlap neighbouring batches' compute
                layer.forward_host_batches(x_hosts[:n], y_hosts[:n], update_bias=True,
                                           logit_offset=off)
            else:
                for j in range(n):
                    layer.forward_host(x_hosts[j], y_hosts[j], update_bias=True,
                                       logit_offset=off)
            done += n

    e2e = {}
    for pipelined in ((True, False) if args.scales == "fp32" else ()):
        layer.forward_host_batches(x_hosts[:1], y_hosts[:1], update_bias=True, logit_offset=off)
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        e2e_steps(pipelined)
        e1.record(st)
        e1.synchronize()
        e2e[pipelined] = max_over_ranks(e0.elapsed_time(e1), world)
    e2e_ms = e2e.get(True)
    xbytes = cfg.T * cfg.d * 2

    # ---- per-batch expert load from the initial bias, batches in order
    # (untimed): max / mean of the counts each batch is routed with
    layer.bias.copy_(bias0)
    per_batch = []
    for j in range(nb):
        layer.forward(batches[j], y, update_bias=True, logit_offset=off)
        c = layer.expert_counts.cpu().numpy()
        per_batch.append(round(float(c.max() / max(c.mean(), 1e-9)), 4))

    # ---- per-stage breakdown (CUDA events on the launching stream)
    brk = stage_breakdown(layer, x, off, args.steps)
    alg = algorithmic_counts(cfg, counts)
    g1_ms = brk["gemm1_swiglu"]
    achieved = alg["gemm1_bytes"] / (g1_ms / 1e3) / 1e9
    hbm_peak = float(peaks["hbm_gbs"])
    fp8_peak_burst = float(peaks["bf16_tflops"]) * FP8_PER_BF16
    fp8_peak_sust = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])) * FP8_PER_BF16
    # the W13 launch is HBM-bound below the ridge (FP8 peak / HBM rate) and
    # tensor-bound above it (the skewed batch: 147,456 rows on 94 experts)
    intensity = alg["flops_gemm1"] / alg["gemm1_bytes"]
    ridge = fp8_peak_burst * 1e12 / (hbm_peak * 1e9)
    rows_total = cfg.T * cfg.topk + cfg.T
    form = moe.moe_grouped_gemm_form(cfg.n_routed + 1, rows_total, 2 * cfg.inter,
                                      moe.MOE_EPI_SWIGLU_QUANT)
    label = (f"grouped_gemm_kernel<{int(form == 2)}, 1> "
             f"({'CTA pairs' if form == 2 else 'single CTAs'}; W13 + SwiGLU + h quant)")
    gemm_forms = {"w13": form,
                  "w2": moe.moe_grouped_gemm_form(cfg.n_routed + 1, rows_total, cfg.d,
                                                  moe.MOE_EPI_F32)}
    if intensity < ridge:
        roofline = {"bound": "hbm", "kernel": label, "achieved": achieved, "peak": hbm_peak,
                    "unit": "GB/s", "frac": achieved / hbm_peak, "peak_source": peak_src,
                    "traffic": profiled_traffic(f"gemm_swiglu_{cfg.name}"),
                    "algorithmic_bytes_per_launch": alg["gemm1_bytes"], "launch_ms": g1_ms}
    else:
        g1_tflops = alg["flops_gemm1"] / (g1_ms / 1e3) / 1e12
        roofline = {"bound": "tensor", "kernel": label, "achieved": g1_tflops,
                    "peak": fp8_peak_burst, "unit": "TFLOP/s", "frac": g1_tflops / fp8_peak_burst,
                    "peak_source": f"{peak_src} bf16 burst x {FP8_PER_BF16:g} (fp8:bf16 nominal)",
                    "traffic": profiled_traffic(f"gemm_swiglu_{cfg.name}"),
                    "algorithmic_flops_per_launch": alg["flops_gemm1"],
                    "algorithmic_bytes_per_launch": alg["gemm1_bytes"], "launch_ms": g1_ms}
    roofline["intensity_flop_per_byte"] = intensity
    roofline["ridge_flop_per_byte"] = ridge
    if roofline["bound"] == "hbm":
        roofline["frac_of_datasheet"] = achieved / DATASHEET["hbm_gbs"]
        roofline["datasheet_peak"] = DATASHEET["hbm_gbs"]
    else:
        roofline["frac_of_datasheet"] = roofline["achieved"] / DATASHEET["fp8_tflops"]
        roofline["datasheet_peak"] = DATASHEET["fp8_tflops"]
    gemm_ms = brk["gemm1_swiglu"] + brk["gemm2"]
    gemm_tflops = alg["layer_flops"] / (gemm_ms / 1e3) / 1e12
    layer_tflops = alg["layer_flops"] * args.steps * world / (ms / 1e3) / 1e12

    line = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp8e4m3/f32" if args.scales == "fp32" else "fp8e4m3+ue8m0/f32",
        "data": "synthetic",
        "config": {"workload": f"moe_layer_{cfg.name}", "scales": args.scales,
                   "T": cfg.T, "d": cfg.d,
                   "n_routed": cfg.n_routed, "n_shared": 1, "n_groups": cfg.n_groups,
                   "topk_groups": cfg.topk_groups, "topk": cfg.topk, "inter": cfg.inter,
                   "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (FP8 expert weights "
                         f"{(cfg.n_routed + 1) * 3 * cfg.d * cfg.inter / 1e9:.1f} GB)"},
        "roofline": roofline,
        "expert_gemm": {"tflops": gemm_tflops, "fp8_peak_tflops": fp8_peak_burst,
                        "ctas_per_tile": gemm_forms,
                        "frac_of_fp8_peak": gemm_tflops / fp8_peak_burst,
                        "frac_of_fp8_sustained": gemm_tflops / fp8_peak_sust,
                        "frac_of_fp8_datasheet": gemm_tflops / DATASHEET["fp8_tflops"],
                        "gemm1_ms": brk["gemm1_swiglu"], "gemm2_ms": brk["gemm2"],
                        "flops_per_step": alg["layer_flops"]},
        "layer_tflops": layer_tflops,
        "breakdown_ms": brk,
        "weight_quant": weight_quant_pass(dev, hbm_peak),
        "memory_passes": memory_passes(cfg, brk, alg, hbm_peak),
        "load": {"max_over_mean": float(counts.max() / max(counts.mean(), 1e-9)),
                 "max_over_mean_per_batch": per_batch,
                 "experts_touched": alg["touched"]},
        "e2e": ({"value": tokens_total / (e2e_ms / 1e3), "unit": "tokens/s",
                 "h2d_bytes_per_step": xbytes, "d2h_bytes_per_step": xbytes,
                 "api": f"moe_layer_forward_host_batches (up to {per_call} batches per call, "
                        "copies overlapped with neighbouring batches' compute)",
                 "unpipelined_value": tokens_total / (e2e[False] / 1e3),
                 "unpipelined_api": "moe_layer_forward_host, one call per step"}
                if e2e else None),
        # route 8, quant+permute 4, GEMMs 2, combine 1, bias update 1
        "gpu_launches": 16 * args.steps,
        "clocks": clk,
        "device_status": status,
    }
    # CPU baseline: the oracle on a bounded sample (rank 0, one GPU only)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        dt, n, cores = oracle_sample_time(cfg, inp, dev, min(CPU_SAMPLE_TOKENS[cfg.name], cfg.T))
        line["cpu_baseline"] = {
            "value": n / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} random tokens of the {cfg.name} batch (routing, quantisation, "
                      "touched experts, combine); weights pre-quantised by the oracle"}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_backward(args, world, rank, local):
    """The layer's backward pass (dx, the router gradient and, unless
    --no-wgrad, the expert weight gradients for an upstream gradient dy) on
    the workload's batch: forward_train once, then timed
    backward calls with dy resident in HBM; beside it end to end with dy
    copied in from pinned host memory and dx copied out every step."""
    import numpy as np
    import torch
    import synthetic as S

    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    cfg = S.CONFIGS[args.workload]
    peaks, peak_src = load_peaks()
    layer, x, off, inp, _ = build_layer(cfg, dev)
    st = torch.cuda.current_stream()
    layer.forward_train(x, logit_offset=off)
    T, d, I, K = cfg.T, cfg.d, cfg.inter, cfg.topk
    dy_host = torch.from_numpy(S.host_normal_bf16(np.random.default_rng(cfg.seed + 100),
                                                  (T, d), 1.0).view(np.int16)).view(
        torch.bfloat16).pin_memory()
    dy = dy_host.to(dev)
    wg = not args.no_wgrad
    for _ in range(args.warmup):
        layer.backward(dy, wgrad=wg)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(dev)
    clocks = ClockSampler(f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local))
    clocks.start()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(st)
    for _ in range(args.steps):
        layer.backward(dy, wgrad=wg)
    ev1.record(st)
    ev1.synchronize()
    clk = clocks.stop()
    barrier(world)
    ms = max_over_ranks(ev0.elapsed_time(ev1), world)
    status = layer.status()
    tokens_total = T * args.steps * world

    # end to end: dy in from pinned host memory, dx out, every step
    dx_host = torch.empty((T, d), dtype=torch.float32).pin_memory()
    dy_dev = torch.empty_like(dy)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(args.steps):
        dy_dev.copy_(dy_host, non_blocking=True)
        dx = layer.backward(dy_dev, wgrad=wg)[0]
        dx_host.copy_(dx, non_blocking=True)
    e1.record(st)
    e1.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)

    # per-stage times (events between the stages, same launches)
    tot = {}
    for it in range(args.steps + 2):
        marks = []
        layer.backward(dy, marks=marks, wgrad=wg)
        marks[-1][1].synchronize()
        if it >= 2:
            for (_, a), (n, b) in zip(marks[:-1], marks[1:]):
                tot[n] = tot.get(n, 0.0) + a.elapsed_time(b)
    brk = {n: v / args.steps for n, v in tot.items()}
    R = T * K + T
    G = cfg.n_routed + 1
    flops = {"gemm_dh": 2.0 * R * d * I, "gemm_ac_recompute": 2.0 * R * d * 2 * I,
             "gemm_dx": 2.0 * R * 2 * I * d}
    # weight gradients: fp32 outputs for every expert (zeros for unchosen ones)
    out_bytes = {}
    if wg:
        flops.update({"gemm_dw13": 2.0 * R * 2 * I * d, "gemm_dw2": 2.0 * R * d * I})
        out_bytes = {"gemm_dw13": 4.0 * G * 2 * I * d, "gemm_dw2": 4.0 * G * d * I}
    top = max(flops, key=lambda n: brk[n])
    fp8_peak = float(peaks["bf16_tflops"]) * FP8_PER_BF16
    hbm_peak = float(peaks["hbm_gbs"])
    ach = flops[top] / (brk[top] / 1e3) / 1e12
    gemm_ms = sum(brk[n] for n in flops)
    if top in out_bytes and out_bytes[top] / (hbm_peak * 1e9) > flops[top] / (fp8_peak * 1e12):
        # the gradient write bounds this launch, not the tensor cores
        gbs = out_bytes[top] / (brk[top] / 1e3) / 1e9
        roof = {"bound": "hbm", "kernel": f"wgrad_gemm_kernel ({top})", "achieved": gbs,
                "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                "peak_source": peak_src, "traffic": None,
                "algorithmic_bytes_per_launch": out_bytes[top], "launch_ms": brk[top],
                "tflops": ach, "frac_of_datasheet": gbs / DATASHEET["hbm_gbs"]}
    else:
        roof = {"bound": "tensor", "kernel": f"grouped GEMM ({top})", "achieved": ach,
                "peak": fp8_peak, "unit": "TFLOP/s", "frac": ach / fp8_peak,
                "peak_source": f"{peak_src} bf16 burst x {FP8_PER_BF16:g}",
                "traffic": None, "algorithmic_flops_per_launch": flops[top],
                "launch_ms": brk[top], "frac_of_datasheet": ach / DATASHEET["fp8_tflops"]}
    mem_bytes = {
        "combine_backward_quant": T * d * 2 + R * d + R * (d // 128) * 4,
        "swiglu_backward_quant": R * I * 4 + R * 2 * I * 4 + R * 2 * I + R * (2 * I // 128) * 4,
        "gate_backward": T * K * d * 4 + T * d * 2,
        "dx_combine": R * d * 4 + T * d * 4 + T * d * 4,
    }
    line = {
        "metric": "backward_tokens_per_s",
        "value": tokens_total / (ms / 1e3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp8e4m3/f32",
        "data": "synthetic",
        "config": {"workload": f"moe_layer_backward_{cfg.name}", "wgrad": wg, "T": T, "d": d,
                   "n_routed": cfg.n_routed, "topk": K, "inter": I,
                   "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (FP8 weights and their transposes, "
                         "fp32 row buffers of several GB)"},
        "roofline": roof,
        "backward_gemms": {n: {"ms": brk[n], "tflops": f / (brk[n] / 1e3) / 1e12,
                               "frac_of_fp8_peak": f / (brk[n] / 1e3) / 1e12 / fp8_peak}
                           for n, f in flops.items()},
        "gemm_tflops": sum(flops.values()) / (gemm_ms / 1e3) / 1e12,
        "memory_passes": {n: {"ms": brk[n], "gbs": b / (brk[n] / 1e3) / 1e9,
                              "frac_of_hbm": b / (brk[n] / 1e3) / 1e9 / hbm_peak}
                          for n, b in mem_bytes.items()},
        "breakdown_ms": brk,
        "e2e": {"value": tokens_total / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": T * d * 2, "d2h_bytes_per_step": T * d * 4,
                "api": "MoeLayer.backward with dy copied in and dx copied out each step"},
        # combine quant 1, GEMMs 3, SwiGLU quant 1, gate 1, router 3, dx 1;
        # weight gradients: layout 1, quantisers 4, GEMMs 2
        "gpu_launches": (17 if wg else 10) * args.steps,
        "clocks": clk,
        "device_status": status,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="skewed",
                    choices=["tiny", "prefill", "decode", "skewed", "prefill_e16", "gemm",
                             "route", "permute", "ep", "redundant"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--scales", choices=["fp32", "ue8m0"], default="fp32",
                    help="fp32: the pages' recipe (default); ue8m0: the power-of-two scale "
                         "option with block-scaled tensor-core GEMMs")
    ap.add_argument("--pass", dest="which", choices=["forward", "backward"], default="forward",
                    help="backward: time the layer's backward pass (dx, router and expert "
                         "weight gradients)")
    ap.add_argument("--no-wgrad", action="store_true",
                    help="backward without the expert weight gradients")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        elif args.workload == "gemm":
            run_gemm(args, world, rank, local)
        elif args.workload == "route":
            run_route(args, world, rank, local)
        elif args.workload == "permute":
            run_permute(args, world, rank, local)
        elif args.workload == "ep":
            run_ep(args, world, rank, local)
        elif args.workload == "redundant":
            run_redundant(args, world, rank, local)
        elif args.which == "backward":
            run_backward(args, world, rank, local)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
