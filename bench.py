#!/usr/bin/env python
"""Benchmark of the NF4 Mixture-of-Experts expert layer: forward + input
gradient (recompute-in-backward) on the OLMoE-1B-7B-shaped layer (E=64, H=2048,
I=1024, top-8 without renormalisation, T=4096 tokens per GPU), NF4 weights with
blocksize-64 fp32 absmax, synthetic seeded inputs.

One step = route (softmax/top-k from fp32 logits) + group + grouped gate_up GEMM
with SwiGLU + grouped down GEMM with the weighted combine + dgrad (two grouped
GEMMs with the weights re-dequantized in-kernel), all through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl e4b|reference]

Prints one JSON line (rank 0).  Multi-GPU: one process per GPU under torchrun,
each GPU runs its own batch (data parallel, no collective on the data path),
value = tokens of all ranks / max-over-ranks device time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "routed tokens/s, NF4 MoE layer fwd+dgrad"
UNIT = "tokens/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="e4b", choices=["e4b", "reference"])
    ap.add_argument("--tokens", type=int, default=4096)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-aux", action="store_true", help="skip the decode and quantize/dequantize legs")
    ap.add_argument("--leg", default="step", choices=["step", "decode", "codec", "variant"],
                    help="step: the benchmark line; decode / codec / variant: only that secondary leg (for profiling), "
                         "decode on the Qwen3-shaped layer at --tokens (default 1)")
    return ap.parse_args()


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank number over all ranks (identity when not distributed).
    NCCL reduces on the rank's GPU, gloo on the host."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    dev = device if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job tokens/s: every rank processes its own batch each step (weak scaling)."""
    return world * tokens_per_rank / (ms_per_step / 1e3)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    for f in ("grouped_gemm.cu", "e4b_device.cuh", "e4b_internal.h"):
        h.update(open(os.path.join(ROOT, "bit_quantized_mixture_nf4_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    src = kernel_source_hash()
    for line in open(path):
        f = line.split()
        if len(f) >= 4 and not line.startswith("#") and f[0] == kernel and f[1] == workload and f[3] == src:
            return float(f[2])
    return None


class ClockSampler:
    """SM clock, power and clock-event (throttle) reasons sampled through NVML by a
    host thread every ~1 ms while the timed region runs (read-only queries)."""
    # NVML clock-event reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_device):
        self.dev = torch_device
        self.samples = []
        self.smax = None
        self._stop = None
        self._thr = None

    def __enter__(self):
        import threading
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            self.smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        except Exception:
            return self
        self._stop = threading.Event()

        def sample():
            try:
                self.samples.append((pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                                     pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0, int(get_reasons(h))))
            except Exception:
                pass

        def loop():
            while not self._stop.is_set():
                sample()
                time.sleep(0.001)
        self._sample = sample
        self._thr = threading.Thread(target=loop, daemon=True)
        self._thr.start()
        return self

    def sample_now(self):
        """One sample from the calling thread (call while the GPU is busy)."""
        if self._thr is not None:
            self._sample()

    def __exit__(self, *a):
        if self._thr is not None:
            self._stop.set()
            self._thr.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.smax, "reasons": ["unsampled"]}
        reasons = set()
        for _, _, r in self.samples:
            for bit, name in self.REASONS.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s[0] for s in self.samples), "sm_max_mhz": self.smax,
                "reasons": sorted(reasons), "samples": len(self.samples),
                "power_w_max": max(s[1] for s in self.samples)}


# ------------------------------------------------------------------ secondary legs

def decode_leg(w, dev, reps=20):
    """Small-batch forward (T <= 8, the weight-streaming GEMV path) on workload w.

    Metric: touched weight bytes / forward time, touched = distinct experts the
    tokens route to x 3*H*I x 0.5625 B.  The layer's packed weights are cycled over
    enough copies (>= 8 and > 4x the L2 size) that every forward streams its
    experts from HBM; the forwards over all copies run as one CUDA graph (route +
    gate_up + down per forward).  Returns a dict for the bench line."""
    import torch
    import bit_quantized_mixture_nf4_b200 as e4b
    from bit_quantized_mixture_nf4_b200 import workloads as wl
    hbm = peaks()[0]
    x = wl.activations(w).to(dev)
    logits = wl.router_logits(w, wl.activations(w)).to(dev)
    gu, dn = wl.weights(w, device=dev)
    pg, ag = e4b.e4b_quantize_nf4(gu, codebook=w.codebook)
    pd, ad = e4b.e4b_quantize_nf4(dn, codebook=w.codebook)
    del gu, dn
    per_layer = pg.numel() + pd.numel() + 4 * (ag.numel() + ad.numel())
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    copies = max(8, -(-4 * l2 // per_layer))
    layers = [(pg, ag, pd, ad)] + [(pg.clone(), ag.clone(), pd.clone(), ad.clone()) for _ in range(copies - 1)]
    experts = [e4b.make_experts(a, c, b, d) for a, b, c, d in layers]
    desc = e4b.make_desc(w.E, w.H, w.I, w.k, w.renorm, w.codebook, 64, e4b.PATH_DECODE)
    idx = torch.empty(w.T, w.k, dtype=torch.int32, device=dev)
    wts = torch.empty(w.T, w.k, dtype=torch.float32, device=dev)
    y = torch.empty(w.T, w.H, dtype=torch.bfloat16, device=dev)
    ws = e4b.workspace(desc, w.T, dev)
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        for ex in experts:                      # warm-up outside the capture
            e4b.e4b_moe_forward(desc, ex, x, logits, idx, wts, y, ws=ws)
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize(dev)
    graph = torch.cuda.CUDAGraph()
    n0 = e4b.e4b_launch_count()
    with torch.cuda.graph(graph):
        for ex in experts:
            e4b.e4b_moe_forward(desc, ex, x, logits, idx, wts, y, ws=ws)
    launches_per_fwd = (e4b.e4b_launch_count() - n0) / copies
    graph.replay()
    torch.cuda.synchronize(dev)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(reps):
        graph.replay()
    e.record()
    torch.cuda.synchronize(dev)
    us = s.elapsed_time(e) * 1e3 / (reps * copies)
    touched = int(torch.unique(idx).numel())
    nbytes = touched * w.weight_bytes_per_expert()
    gbs = nbytes / (us * 1e-6) / 1e9
    del graph
    if e4b.e4b_device_status() != e4b.E4B_OK:
        raise RuntimeError("device status not ok after the decode leg")
    return {"workload": f"{w.name}-shaped E={w.E} H={w.H} I={w.I} top{w.k} T={w.T} "
                        f"{'fp4' if w.codebook else 'nf4'}", "us_per_forward": us,
            "experts_touched": touched, "bytes_per_forward": nbytes, "weight_stream_gbs": gbs,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm},
            "layer_copies": copies, "kernels_per_forward": launches_per_fwd, "timing": "CUDA graph, events"}


def variant_leg(w, dev, reps=10):
    """The gpt-oss expert variant (per-expert biases, clamped GLU alpha 1.702 and
    limit 7) on workload w: forward (routed from logits, derivatives saved) plus
    input gradient, L2 flushed between steps; tokens/s and the whole step against
    the dense-bf16 peak (12*H*I FLOP per pair)."""
    import torch
    import bit_quantized_mixture_nf4_b200 as e4b
    from bit_quantized_mixture_nf4_b200 import workloads as wl
    bf16 = peaks()[1]
    x = wl.activations(w).to(dev)
    logits = wl.router_logits(w, wl.activations(w)).to(dev)
    go = wl.grad_output(w).to(dev)
    gu, dn = wl.weights(w, device=dev)
    pg, ag = e4b.e4b_quantize_nf4(gu, codebook=w.codebook)
    pd, ad = e4b.e4b_quantize_nf4(dn, codebook=w.codebook)
    del gu, dn
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed + 7)
    bgu = torch.randn(w.E, 2 * w.I, device=dev, generator=g) * 0.3
    bd = torch.randn(w.E, w.H, device=dev, generator=g) * 0.3
    experts = e4b.make_experts(pg, pd, ag, ad, bgu, bd)
    desc = e4b.make_desc(w.E, w.H, w.I, w.k, w.renorm, w.codebook, 64, e4b.PATH_GROUPED, e4b.ACT_CLAMPED_GLU,
                         1.702, 7.0)
    P = w.T * w.k
    idx = torch.empty(w.T, w.k, dtype=torch.int32, device=dev)
    wts = torch.empty(w.T, w.k, dtype=torch.float32, device=dev)
    y = torch.empty(w.T, w.H, dtype=torch.bfloat16, device=dev)
    gx = torch.empty(w.T, w.H, dtype=torch.bfloat16, device=dev)
    saved = torch.empty(P, 2 * w.I, dtype=torch.bfloat16, device=dev)
    ws = e4b.workspace(desc, w.T, dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def step():
        e4b.e4b_moe_forward(desc, experts, x, logits, idx, wts, y, saved_gu=saved, ws=ws)
        e4b.e4b_moe_backward_dgrad(desc, experts, x, idx, wts, go, saved_gu=saved, grad_x=gx, ws=ws)

    for _ in range(3):
        step()
    torch.cuda.synchronize(dev)
    ss = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
    ee = [torch.cuda.Event(enable_timing=True) for _ in range(reps)]
    for i in range(reps):
        flush.zero_()
        ss[i].record()
        step()
        ee[i].record()
    torch.cuda.synchronize(dev)
    ms = sum(a.elapsed_time(b) for a, b in zip(ss, ee)) / reps
    if e4b.e4b_device_status() != e4b.E4B_OK:
        raise RuntimeError("device status not ok after the variant leg")
    tf = 12 * w.H * w.I * P / (ms / 1e3) / 1e12
    return {"workload": f"{w.name}-shaped E={w.E} H={w.H} I={w.I} top{w.k} T={w.T} "
                        f"{'fp4' if w.codebook else 'nf4'}, clamped GLU + per-expert biases, fwd + dgrad",
            "ms_per_step": ms, "tokens_per_s": w.T / (ms / 1e3),
            "roofline": {"bound": "tensor", "achieved": tf, "peak": bf16, "unit": "TFLOP/s", "frac": tf / bf16},
            "l2": "flushed between steps"}


def codec_leg(w, dev, reps=10):
    """Standalone quantize (fp32 -> packed + absmax) and bf16 dequantize over the
    whole gate_up stack of workload w; HBM-bound: quantize moves 4 + 0.5625 B and
    dequantize 0.5625 + 2 B per weight element."""
    import torch
    import bit_quantized_mixture_nf4_b200 as e4b
    from bit_quantized_mixture_nf4_b200 import workloads as wl
    hbm = peaks()[0]
    gu, _ = wl.weights(w, device=dev)
    n = gu.numel()
    packed = torch.empty(n // 2, dtype=torch.uint8, device=dev)
    absmax = torch.empty(n // 64, dtype=torch.float32, device=dev)
    out = torch.empty(n, dtype=torch.bfloat16, device=dev)
    shape = tuple(gu.shape)

    def q():
        e4b.e4b_quantize_nf4(gu, codebook=w.codebook, packed=packed, absmax=absmax)

    def dq():
        e4b.e4b_dequantize_nf4(packed, absmax, shape, codebook=w.codebook, out_dtype=e4b.BF16, out=out)

    res = {}
    for name, fn, bpe in (("quantize", q, 4.5625), ("dequantize", dq, 2.5625)):
        for _ in range(3):
            fn()
        torch.cuda.synchronize(dev)
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(reps):
            fn()
        e.record()
        torch.cuda.synchronize(dev)
        us = s.elapsed_time(e) * 1e3 / reps
        gbs = n * bpe / (us * 1e-6) / 1e9
        res[name] = {"elements": n, "us": us, "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                     "bytes_per_element": bpe}
    res["workload"] = f"{w.name}-shaped gate_up stack [{w.E},{2 * w.I},{w.H}] {'fp4' if w.codebook else 'nf4'}"
    del gu, out
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------------ CPU oracle

def oracle_step(w, x, logits, go, packed, sample_tokens, dequant_cache):
    """One oracle pass: route + group all tokens, dequantize the experts (from the
    packed bytes), forward + input gradient of the sampled tokens.  Returns
    (seconds for the whole-batch fixed part, seconds for the sampled tokens)."""
    import numpy as np
    import oracle
    t0 = time.perf_counter()
    idx, wts = oracle.route(logits, w.k, w.renorm)
    oracle.permute(idx, w.E)
    pg, ag, pd, ad = packed
    wgu = oracle.dequantize(pg, ag, (w.E, 2 * w.I, w.H), w.codebook)
    wd = oracle.dequantize(pd, ad, (w.E, w.H, w.I), w.codebook)
    t1 = time.perf_counter()
    toks = np.asarray(sample_tokens, np.int64)
    oracle.forward(x, idx, wts, wgu, wd, tokens=toks)
    oracle.dgrad(x, go, idx, wts, wgu, wd, tokens=toks)
    t2 = time.perf_counter()
    return t1 - t0, t2 - t1


def oracle_inputs(w):
    import oracle
    from bit_quantized_mixture_nf4_b200 import workloads as wl
    x = wl.activations(w)
    gu, dn = wl.weights(w)
    logits = wl.router_logits(w, x).numpy()
    go = wl.grad_output(w).float().numpy()
    packed = oracle.quantize(gu.numpy(), w.codebook) + oracle.quantize(dn.numpy(), w.codebook)
    return x.float().numpy(), logits, go, packed


def cpu_rate(w, target_s=12.0, inputs=None):
    """Oracle throughput in routed tokens/s on a bounded sample, scaled to a full batch."""
    import numpy as np
    import oracle
    x, logits, go, packed = inputs if inputs is not None else oracle_inputs(w)
    nth = oracle.num_threads()
    rng = np.random.default_rng(0)
    cal = rng.choice(w.T, size=min(w.T, nth), replace=False)
    fixed, tcal = oracle_step(w, x, logits, go, packed, cal, None)
    per_tok = tcal / len(cal)
    S = int(max(len(cal), min(w.T, (target_s - fixed) / max(per_tok, 1e-9))))
    S = max(nth, (S // nth) * nth)
    toks = rng.choice(w.T, size=min(S, w.T), replace=False)
    fixed, ttok = oracle_step(w, x, logits, go, packed, toks, None)
    step = fixed + ttok * w.T / len(toks)
    return w.T / step, dict(cores=nth, sample=f"{len(toks)} of {w.T} tokens (fwd+dgrad), whole-batch routing, "
                                               f"grouping and dequantization; step time extrapolated linearly in "
                                               f"tokens", fixed_s=fixed, sample_s=ttok)


def run_reference(args, w):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    inputs = oracle_inputs(w)
    import numpy as np
    import oracle
    nth = oracle.num_threads()
    rng = np.random.default_rng(1)
    S = max(nth, 2 * nth)
    toks = rng.choice(w.T, size=min(S, w.T), replace=False)
    for _ in range(args.warmup):
        oracle_step(w, *inputs, toks, None)
    steps = []
    for _ in range(args.steps):
        fixed, ttok = oracle_step(w, *inputs, toks, None)
        steps.append(fixed + ttok * w.T / len(toks))
    step = statistics.median(steps)
    value = w.T / step
    sample = (f"{len(toks)} of {w.T} tokens per step (fwd+dgrad), whole-batch routing, grouping and "
              f"dequantization; step time extrapolated linearly in tokens")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"olmoe-shaped E={w.E} H={w.H} I={w.I} top{w.k} T={w.T} nf4 fwd+dgrad",
                       "global_batch": w.T * world, "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": nth, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm

def run_e4b(args, w):
    import torch
    import bit_quantized_mixture_nf4_b200 as e4b
    from bit_quantized_mixture_nf4_b200 import workloads as wl

    world, rank, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    # inputs: activations / logits / grad_out drawn on the host (seeded), weights on the device
    x_h = wl.activations(w)
    logits_h = wl.router_logits(w, x_h)
    go_h = wl.grad_output(w)
    gu, dn = wl.weights(w, device=dev)
    pg, ag = e4b.e4b_quantize_nf4(gu, codebook=w.codebook)
    pd, ad = e4b.e4b_quantize_nf4(dn, codebook=w.codebook)
    del gu, dn
    torch.cuda.empty_cache()
    experts = e4b.make_experts(pg, pd, ag, ad)
    desc = e4b.make_desc(w.E, w.H, w.I, w.k, w.renorm, w.codebook, 64, e4b.PATH_AUTO)
    T, P = w.T, w.P
    x = x_h.to(dev)
    logits = logits_h.to(dev)
    go = go_h.to(dev)
    idx = torch.empty(T, w.k, dtype=torch.int32, device=dev)
    wts = torch.empty(T, w.k, dtype=torch.float32, device=dev)
    y = torch.empty(T, w.H, dtype=torch.bfloat16, device=dev)
    gx = torch.empty(T, w.H, dtype=torch.bfloat16, device=dev)
    saved = torch.empty(P, 2 * w.I, dtype=torch.bfloat16, device=dev)
    ws = e4b.workspace(desc, T, dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)   # > 126 MB L2
    stream = torch.cuda.current_stream()

    def step():
        e4b.e4b_moe_forward(desc, experts, x, logits, idx, wts, y, saved_gu=saved, ws=ws, stream=stream)
        e4b.e4b_moe_backward_dgrad(desc, experts, x, idx, wts, go, saved_gu=saved, grad_x=gx, ws=ws, stream=stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    if e4b.e4b_device_status() != e4b.E4B_OK:
        raise RuntimeError("device status not ok after warm-up")

    # ------------------------------------------------ device-timed region
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e4b.e4b_timing_reset()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    launches0 = e4b.e4b_launch_count()
    gemm_kinds = ("gemm_gateup", "gemm_down", "gemm_dgrad_down", "gemm_dgrad_gateup")
    with ClockSampler(dev) as clk:
        # only the grouped GEMMs carry events inside the timed region; the small
        # kernels between them run back to back (their breakdown is taken below)
        e4b.e4b_timing_enable_kinds(gemm_kinds)
        for i in range(args.steps):
            flush.zero_()                       # evict L2 between timed steps (not timed)
            starts[i].record(stream)
            step()
            ends[i].record(stream)
            if i % 8 == 7:
                clk.sample_now()                # the queued steps keep the GPU busy meanwhile
        torch.cuda.synchronize()
        e4b.e4b_timing_enable(False)
    launches = e4b.e4b_launch_count() - launches0
    if world > 1:
        torch.distributed.barrier()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = max_over_ranks(sum(step_ms), dev)
    ms_per_step = total_ms / args.steps
    value = job_throughput(T, world, ms_per_step)

    kernels = {}
    for name in gemm_kinds:
        ms, n = e4b.e4b_timing_get(name)
        if n:
            kernels[name] = {"launches": n, "avg_ms": ms / n}

    # per-kernel breakdown of the rest of the step: a short separate pass with every
    # kind bracketed by events (which serialises the chained small kernels)
    e4b.e4b_timing_reset()
    e4b.e4b_timing_enable(True)
    for _ in range(5):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    e4b.e4b_timing_enable(False)
    small_kernels = {}
    for name in ("route", "group", "gather", "combine"):
        ms, n = e4b.e4b_timing_get(name)
        if n:
            small_kernels[name] = {"launches": n, "avg_ms": ms / n}
    flops = {"gemm_gateup": 4, "gemm_down": 2, "gemm_dgrad_down": 2, "gemm_dgrad_gateup": 4}
    dom = max((k for k in flops if k in kernels), key=lambda k: kernels[k]["avg_ms"] * kernels[k]["launches"])
    hbm, bf16_burst, bf16_sus, peak_src = peaks()
    dom_flops = flops[dom] * w.H * w.I * P
    achieved = dom_flops / (kernels[dom]["avg_ms"] / 1e3) / 1e12
    wl_name = f"olmoe_T{T}"
    traffic = recorded_traffic(dom, wl_name)

    # ------------------------------------------------ end-to-end through host buffers
    # The C-ABI's pipelined host-buffer runner: every step copies its inputs in
    # from pinned host memory and its y and grad_x out, on copy streams that
    # overlap one batch's copies with the neighbouring batches' kernels.
    e2e = None
    if not args.no_e2e:
        x_p = x_h.pin_memory()
        l_p = logits_h.pin_memory()
        g_p = go_h.pin_memory()
        y_p = torch.empty(T, w.H, dtype=torch.bfloat16).pin_memory()
        gx_p = torch.empty(T, w.H, dtype=torch.bfloat16).pin_memory()
        pipe = e4b.e4b_pipe_create(desc, experts, T, dev, stream)
        try:
            for _ in range(3):
                e4b.e4b_pipe_submit(pipe, x_p, l_p, g_p, y_p, gx_p)
            e4b.e4b_pipe_sync(pipe)
            if world > 1:
                torch.distributed.barrier()
            es, ee = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            es.record(stream)
            e4b.e4b_pipe_join(pipe)          # the pipe's copies start after es
            for _ in range(args.steps):
                e4b.e4b_pipe_submit(pipe, x_p, l_p, g_p, y_p, gx_p)
            e4b.e4b_pipe_join(pipe)          # ee after the last copy out
            ee.record(stream)
            e4b.e4b_pipe_sync(pipe)
            torch.cuda.synchronize()
        finally:
            e4b.e4b_pipe_destroy(pipe)
        e2e_ms = max_over_ranks(es.elapsed_time(ee) / args.steps, dev)
        h2d = x_p.numel() * 2 + l_p.numel() * 4 + g_p.numel() * 2
        d2h = y_p.numel() * 2 + gx_p.numel() * 2
        e2e = {"value": job_throughput(T, world, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "api": "e4b_pipe_submit (pinned host buffers; copies of one batch overlap the kernels of the "
                      "neighbouring batches)"}

    if e4b.e4b_device_status() != e4b.E4B_OK:
        raise RuntimeError("device status not ok after the timed region")

    # ------------------------------------------------ routing gradient (the other half of the backward)
    aux = {}
    if not args.no_aux:
        dwt = torch.empty(T, w.k, dtype=torch.float32, device=dev)
        dlg = torch.empty(T, w.E, dtype=torch.float32, device=dev)

        def rstep():
            e4b.e4b_moe_backward_router(desc, experts, x, idx, wts, go, router_logits=logits, grad_topk_w=dwt,
                                        grad_logits=dlg, ws=ws, stream=stream)

        for _ in range(3):
            rstep()
        torch.cuda.synchronize()
        rs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        re_ = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        for i in range(args.steps):
            flush.zero_()
            rs[i].record(stream)
            rstep()
            re_[i].record(stream)
        torch.cuda.synchronize()
        r_ms = sum(a.elapsed_time(b) for a, b in zip(rs, re_)) / args.steps
        r_flops = 6 * w.H * w.I * P
        aux["router_backward"] = {
            "workload": f"same layer and batch as the step (T={T})", "us": r_ms * 1e3,
            "roofline": {"bound": "tensor", "achieved": r_flops / (r_ms / 1e3) / 1e12, "peak": bf16_burst,
                         "unit": "TFLOP/s", "frac": r_flops / (r_ms / 1e3) / 1e12 / bf16_burst},
            "work": "h and the unweighted expert outputs recomputed by the grouped GEMMs (6*H*I FLOP per pair), "
                    "then one fp32 dot product per pair and the softmax backward per token"}
        del dwt, dlg

    # ------------------------------------------------ secondary legs (small-batch decode, codec)
    if not args.no_aux:
        del saved, ws
        torch.cuda.empty_cache()
        aux["decode"] = [decode_leg(v, dev) for v in (wl.QWEN3.with_tokens(1), wl.GPTOSS.with_tokens(1),
                                                      wl.QWEN3.with_tokens(8))]
        torch.cuda.empty_cache()
        aux["codec"] = codec_leg(wl.OLMOE, dev)
        torch.cuda.empty_cache()
        aux["gptoss_variant"] = variant_leg(wl.GPTOSS.with_tokens(2048), dev)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, info = cpu_rate(w)
        cpu = {"value": rate, "unit": UNIT, "cores": info["cores"], "kind": "oracle", "sample": info["sample"]}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"olmoe-shaped E={w.E} H={w.H} I={w.I} top{w.k} no-renorm T={T}/GPU, nf4 "
                                   f"blocksize 64, fwd (routed from logits, g/u saved) + dgrad",
                       "global_batch": T * world, "parallelism": f"dp{world} (independent batches)",
                       "l2": "flushed between timed steps (256 MB write)", "routed_pairs_per_gpu": P},
            "roofline": {"kernel": dom, "bound": "tensor", "achieved": achieved, "peak": bf16_burst,
                         "unit": "TFLOP/s", "frac": achieved / bf16_burst, "traffic": traffic,
                         "peak_kind": f"{peak_src} bf16 dense (burst)",
                         "flops_per_launch": dom_flops, "avg_launch_ms": kernels[dom]["avg_ms"]},
            "kernels": kernels,
            "small_kernels": {"timed": "separate 5-step pass, every launch bracketed by events", **small_kernels},
            "clocks": clk.summary(),
            "gpu_launches": launches,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        line.update(aux)
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def main():
    args = parse()
    from bit_quantized_mixture_nf4_b200 import workloads as wl
    if args.leg != "step":
        import torch
        dev = torch.device("cuda", 0)
        if args.leg == "decode":
            tokens = args.tokens if args.tokens <= 8 else 1
            print(json.dumps(decode_leg(wl.QWEN3.with_tokens(tokens), dev, reps=max(args.steps, 3))), flush=True)
        elif args.leg == "variant":
            print(json.dumps(variant_leg(wl.GPTOSS.with_tokens(2048), dev, reps=max(args.steps, 3))), flush=True)
        else:
            print(json.dumps(codec_leg(wl.OLMOE, dev, reps=max(args.steps, 3))), flush=True)
        return
    w = wl.OLMOE.with_tokens(args.tokens)
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_e4b(args, w)


if __name__ == "__main__":
    main()
