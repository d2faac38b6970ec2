#!/usr/bin/env python
"""Benchmark of the NF4 Mixture-of-Experts expert layer.

Headline: one training step (forward routed from fp32 logits + the input
gradient with the weights re-dequantized in-kernel) of the Mixtral-8x7B-shaped
layer (E=8, H=4096, I=14336, top-2 renormalised, T=16384 tokens per GPU), NF4
weights with blocksize-64 fp32 absmax, synthetic seeded inputs, through the C
ABI.  Metric: routed tokens/s of forward + input gradient; the dominant kernel
and the whole step are reported against the dense-bf16 tensor peak
(12*H*I FLOP per routed pair for a step).

Secondary legs on the same line: the other large layers (OLMoE T=4096, Qwen3
prefill T=8192 with Zipf-skewed routing, gpt-oss FP4 T=2048), the small-batch
decode path (Qwen3 T=1,2,4,8 and gpt-oss T=1: touched weight bytes / time
against HBM peak), the routing gradient, the gpt-oss expert variant, the
standalone codec kernels and the NF4-vs-FP4 reconstruction error of the
gpt-oss-shaped stacks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl e4b|reference]

Prints one JSON line (rank 0).  Multi-GPU: one process per GPU under torchrun,
each GPU runs its own batch (data parallel, no collective on the data path),
value = tokens of all ranks / max-over-ranks device time.
"""
from __future__ import annotations

import argparse
import dataclasses
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
GEMM_FLOPS = {"gemm_gateup": 4, "gemm_down": 2, "gemm_dgrad_down": 2, "gemm_dgrad_gateup": 4}   # x H*I per pair


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="e4b", choices=["e4b", "reference"])
    ap.add_argument("--workload", default="mixtral", choices=["mixtral", "olmoe", "qwen3", "gptoss"],
                    help="layer of the headline step (default: the Mixtral-shaped layer, the largest config)")
    ap.add_argument("--tokens", type=int, default=0, help="tokens per GPU (0: the workload's own T)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-aux", action="store_true", help="skip the secondary legs")
    ap.add_argument("--codebook", default="native", choices=["native", "mxfp4"],
                    help="variant leg: the workload's own 4-bit codebook or native MXFP4 storage")
    ap.add_argument("--leg", default="step",
                    choices=["step", "decode", "codec", "variant", "router", "lora", "storage"],
                    help="step: the benchmark line; decode / codec / variant / router: only that secondary leg "
                         "(for profiling); decode runs the Qwen3-shaped layer (or --workload) at --tokens "
                         "(default 1); router runs the routing-gradient legs on --workload")
    return ap.parse_args()


def headline_workload(args):
    from bit_quantized_mixture_nf4_b200 import workloads as wl
    w = wl.ALL[args.workload]
    return w.with_tokens(args.tokens) if args.tokens > 0 else w


def workload_desc(w) -> str:
    rt = "zipf-skewed routing, " if w.router == "zipf" else ""
    return (f"{w.name}-shaped E={w.E} H={w.H} I={w.I} top{w.k} {'renorm' if w.renorm else 'no-renorm'} T={w.T}/GPU, "
            f"{('nf4', 'fp4', 'mxfp4', 'int8', 'fp8', 'bf16')[w.codebook]} blocksize {32 if w.codebook == 2 else 64}, {rt}fwd (routed from logits, g/u saved) + dgrad")


def bench_config(w, world):
    """The config dict both arms print for the headline workload."""
    return {"workload": workload_desc(w), "global_batch": w.T * world, "routed_pairs_per_gpu": w.P,
            "parallelism": f"dp{world} (independent batches)",
            "l2": "flushed between timed steps (256 MB write)"}


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


def pct(values, q):
    """q-th percentile (0..100) by linear interpolation."""
    v = sorted(values)
    if not v:
        return None
    pos = (len(v) - 1) * q / 100.0
    lo = int(pos)
    hi = min(lo + 1, len(v) - 1)
    return v[lo] + (v[hi] - v[lo]) * (pos - lo)


def step_stats(ms):
    return {"median": statistics.median(ms), "p10": pct(ms, 10), "p90": pct(ms, 90), "mean": sum(ms) / len(ms),
            "n": len(ms)}


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


# ------------------------------------------------------------------ GPU layer set-up

class Layer:
    """One quantized layer on the device with its seeded inputs (drawn on the host,
    so the CPU oracle can be fed the same values) and output buffers."""

    def __init__(self, w, dev, path=0, act=0, biases=False, lora_rank=0):
        import torch
        import bit_quantized_mixture_nf4_b200 as e4b
        from bit_quantized_mixture_nf4_b200 import workloads as wl
        self.w, self.dev = w, dev
        self.x_h = wl.activations(w)
        self.logits_h = wl.router_logits(w, self.x_h)
        self.go_h = wl.grad_output(w)
        gu, dn = wl.weights(w, device=dev)
        self.mx = w.codebook == wl.MXFP4   # native MXFP4: packed codes + E8M0 scale bytes
        if self.mx:
            quant = e4b.e4b_quantize_mxfp4
        elif w.codebook == wl.BF16_WEIGHTS:   # passthrough: the bf16 stacks themselves, no absmax
            quant = lambda t: (t.to(torch.bfloat16).view(torch.uint8).reshape(t.shape[0], -1), None)
        else:
            quant = lambda t: e4b.e4b_quantize_nf4(t, codebook=w.codebook)
        self.pg, self.ag = quant(gu)
        self.pd, self.ad = quant(dn)
        del gu, dn
        self.bgu = self.bd = None
        if biases:
            g = torch.Generator(device=dev)
            g.manual_seed(w.seed + 7)
            self.bgu = torch.randn(w.E, 2 * w.I, device=dev, generator=g) * 0.3
            self.bd = torch.randn(w.E, w.H, device=dev, generator=g) * 0.3
        self.lora = self.lora_grads = None
        if lora_rank:   # per-expert adapters (A ~ N(0, 1/in), B ~ N(0, 0.01/r)), bf16
            g = torch.Generator(device=dev)
            g.manual_seed(w.seed + 11)
            r = lora_rank
            shapes = ((w.E, r, w.H, 1 / w.H), (w.E, 2 * w.I, r, 0.01 / r), (w.E, r, w.I, 1 / w.I),
                      (w.E, w.H, r, 0.01 / r))
            self.lora = tuple((torch.randn(a, b, c, device=dev, generator=g) * v ** 0.5).to(torch.bfloat16)
                              for a, b, c, v in shapes)
            self.lora_grads = tuple(torch.empty(t.shape, dtype=torch.float32, device=dev) for t in self.lora)
        if self.mx:
            self.experts = e4b.make_experts(self.pg, self.pd, None, None, self.bgu, self.bd, lora=self.lora,
                                            gate_up_scales=self.ag, down_scales=self.ad)
        else:
            self.experts = e4b.make_experts(self.pg, self.pd, self.ag, self.ad, self.bgu, self.bd, lora=self.lora)
        self.desc = e4b.make_desc(w.E, w.H, w.I, w.k, w.renorm, w.codebook, 32 if self.mx else 64, path, act, 1.702,
                                  7.0, lora_rank=lora_rank, lora_scale=2.0)
        T, P = w.T, w.P
        self.x = self.x_h.to(dev)
        self.logits = self.logits_h.to(dev)
        self.go = self.go_h.to(dev)
        self.idx = torch.empty(T, w.k, dtype=torch.int32, device=dev)
        self.wts = torch.empty(T, w.k, dtype=torch.float32, device=dev)
        self.y = torch.empty(T, w.H, dtype=torch.bfloat16, device=dev)
        self.gx = torch.empty(T, w.H, dtype=torch.bfloat16, device=dev)
        self.saved = torch.empty(P, 2 * w.I, dtype=torch.bfloat16, device=dev)
        self.ws = e4b.workspace(self.desc, T, dev)
        self.routing = False   # True: the step also takes the routing gradient (fused backward)
        self.saved_h = self.dwt = self.dlg = None
        torch.cuda.empty_cache()

    def with_routing_gradient(self):
        """Switch the step to forward (saving h) + the one-pass layer backward with
        grad_x, grad_topk_w and grad_logits."""
        import torch
        w, dev = self.w, self.dev
        self.saved_h = torch.empty(w.P, w.I, dtype=torch.bfloat16, device=dev)
        self.dwt = torch.empty(w.T, w.k, dtype=torch.float32, device=dev)
        self.dlg = torch.empty(w.T, w.E, dtype=torch.float32, device=dev)
        self.routing = True

    def step(self, stream=None):
        import bit_quantized_mixture_nf4_b200 as e4b
        e4b.e4b_moe_forward(self.desc, self.experts, self.x, self.logits, self.idx, self.wts, self.y,
                            saved_gu=self.saved, ws=self.ws, stream=stream, saved_h=self.saved_h)
        if self.routing or self.lora is not None:
            e4b.e4b_moe_backward(self.desc, self.experts, self.x, self.idx, self.wts, self.go, saved_gu=self.saved,
                                 saved_h=self.saved_h, router_logits=self.logits if self.routing else None,
                                 grad_x=self.gx, grad_topk_w=self.dwt, grad_logits=self.dlg,
                                 want_routing=self.routing, lora_grads=self.lora_grads, ws=self.ws, stream=stream)
        else:
            e4b.e4b_moe_backward_dgrad(self.desc, self.experts, self.x, self.idx, self.wts, self.go,
                                       saved_gu=self.saved, grad_x=self.gx, ws=self.ws, stream=stream)


def timed_steps(layer, steps, warmup, flush, stream, clk=None, kinds=tuple(GEMM_FLOPS)):
    """Per-step device times (ms) of `steps` fwd+dgrad steps after `warmup` untimed
    ones, L2 flushed between steps; the grouped GEMMs carry per-launch events."""
    import torch
    import bit_quantized_mixture_nf4_b200 as e4b
    for _ in range(max(warmup, 3)):
        layer.step(stream)
    torch.cuda.synchronize()
    if e4b.e4b_device_status() != e4b.E4B_OK:
        raise RuntimeError("device status not ok after warm-up")
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    e4b.e4b_timing_reset()
    torch.cuda.synchronize()
    n0 = e4b.e4b_launch_count()
    e4b.e4b_timing_enable_kinds(kinds)
    for i in range(steps):
        flush.zero_()                       # evict L2 between timed steps (not timed)
        starts[i].record(stream)
        layer.step(stream)
        ends[i].record(stream)
        if clk is not None and i % 4 == 3:
            clk.sample_now()                # the queued steps keep the GPU busy meanwhile
    torch.cuda.synchronize()
    e4b.e4b_timing_enable(False)
    launches = e4b.e4b_launch_count() - n0
    ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    kernels = {}
    for name in kinds:
        t, n = e4b.e4b_timing_get(name)
        if n:
            kernels[name] = {"launches": n, "avg_ms": t / n}
    if e4b.e4b_device_status() != e4b.E4B_OK:
        raise RuntimeError("device status not ok after the timed steps")
    return ms, kernels, launches


def roofline_peak(loop_ms, burst, sustained, source):
    """(peak TFLOP/s, description) for GEMMs timed inside a step loop of loop_ms.  A
    loop that runs for a quarter of a second or more runs under the board's power cap,
    so the sustained dense-bf16 figure is the denominator there; a short loop (or no
    sustained figure) uses the burst one."""
    if sustained is not None and loop_ms >= 250.0:
        return sustained, f"{source} bf16 dense (sustained): timed inside a {loop_ms / 1e3:.2f} s step loop"
    return burst, f"{source} bf16 dense (burst)"


def gemm_roofline(w, kernels, bf16, peak_kind, bf16_burst=None):
    """The dominant grouped GEMM (largest total time) against the dense-bf16 peak `bf16`
    (the burst figure, or the sustained one for kernels timed inside a long step loop;
    bf16_burst given: the fraction of the burst figure is reported beside it)."""
    dom = max((k for k in GEMM_FLOPS if k in kernels), key=lambda k: kernels[k]["avg_ms"] * kernels[k]["launches"])
    flops = GEMM_FLOPS[dom] * w.H * w.I * w.P
    achieved = flops / (kernels[dom]["avg_ms"] / 1e3) / 1e12

    def entry(k, v):
        tf = GEMM_FLOPS[k] * w.H * w.I * w.P / (v["avg_ms"] / 1e3) / 1e12
        e = {"avg_ms": v["avg_ms"], "tflops": tf, "frac": tf / bf16}
        if bf16_burst:
            e["frac_of_burst"] = tf / bf16_burst
        return e

    per_kernel = {k: entry(k, v) for k, v in kernels.items() if k in GEMM_FLOPS}
    roof = {"kernel": dom, "bound": "tensor", "achieved": achieved, "peak": bf16, "unit": "TFLOP/s",
            "frac": achieved / bf16, "peak_kind": peak_kind, "flops_per_launch": flops,
            "avg_launch_ms": kernels[dom]["avg_ms"]}
    if bf16_burst:
        roof["frac_of_burst"] = achieved / bf16_burst
    return roof, per_kernel


# ------------------------------------------------------------------ secondary legs

def step_leg(w, dev, flush, steps=10):
    """fwd+dgrad of another large layer: tokens/s, whole step and dominant GEMM vs dense bf16."""
    import torch
    _, bf16, _, src = peaks()
    layer = Layer(w, dev)
    stream = torch.cuda.current_stream()
    ms, kernels, _ = timed_steps(layer, steps, 3, flush, stream)
    st = step_stats(ms)
    roof, per_kernel = gemm_roofline(w, kernels, bf16, f"{src} bf16 dense (burst)")
    step_tf = 12 * w.H * w.I * w.P / (st["median"] / 1e3) / 1e12
    del layer
    torch.cuda.empty_cache()
    return {"workload": workload_desc(w), "tokens_per_s": w.T / (st["median"] / 1e3), "step_ms": st,
            "step_roofline": {"bound": "tensor", "achieved": step_tf, "peak": bf16, "unit": "TFLOP/s",
                              "frac": step_tf / bf16, "flops_per_step": 12 * w.H * w.I * w.P},
            "roofline": roof, "kernels": per_kernel}


def decode_leg(w, dev, reps=20):
    """Small-batch forward (T <= 8, the weight-streaming decode kernels) on workload w.

    Metric: touched weight bytes / forward time, touched = distinct experts the
    tokens route to x 3*H*I x 0.5625 B.  The layer's packed weights are cycled
    over enough copies that the TOUCHED bytes of all copies exceed 4x the L2 (and
    at least 8 copies), so every forward streams its experts from HBM; the
    forwards over all copies run as one CUDA graph (routing + gate_up + down per
    forward)."""
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
    desc = e4b.make_desc(w.E, w.H, w.I, w.k, w.renorm, w.codebook, 64, e4b.PATH_DECODE)
    idx = torch.empty(w.T, w.k, dtype=torch.int32, device=dev)
    wts = torch.empty(w.T, w.k, dtype=torch.float32, device=dev)
    y = torch.empty(w.T, w.H, dtype=torch.bfloat16, device=dev)
    ws = e4b.workspace(desc, w.T, dev)
    e4b.e4b_moe_forward(desc, e4b.make_experts(pg, pd, ag, ad), x, logits, idx, wts, y, ws=ws)
    torch.cuda.synchronize()
    touched = int(torch.unique(idx).numel())
    nbytes = touched * w.weight_bytes_per_expert()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    copies = max(8, -(-4 * l2 // int(nbytes)))
    layers = [(pg, ag, pd, ad)] + [(pg.clone(), ag.clone(), pd.clone(), ad.clone()) for _ in range(copies - 1)]
    experts = [e4b.make_experts(a, c, b, d) for a, b, c, d in layers]
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
    us = []
    for _ in range(reps):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        graph.replay()
        e.record()
        torch.cuda.synchronize(dev)
        us.append(s.elapsed_time(e) * 1e3 / copies)
    st = step_stats(us)
    gbs = nbytes / (st["median"] * 1e-6) / 1e9
    del graph
    if e4b.e4b_device_status() != e4b.E4B_OK:
        raise RuntimeError("device status not ok after the decode leg")
    return {"workload": f"{w.name}-shaped E={w.E} H={w.H} I={w.I} top{w.k} T={w.T} "
                        f"{('nf4', 'fp4', 'mxfp4', 'int8', 'fp8', 'bf16')[w.codebook]}", "us_per_forward": st,
            "experts_touched": touched, "bytes_per_forward": nbytes, "weight_stream_gbs": gbs,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm},
            "layer_copies": copies, "touched_bytes_all_copies": nbytes * copies,
            "kernels_per_forward": launches_per_fwd, "timing": "CUDA graph over all copies, events, median of reps"}


def variant_leg(w, dev, flush, steps=10):
    """The gpt-oss expert variant (per-expert biases, clamped GLU alpha 1.702 and
    limit 7) on workload w: forward + input gradient, L2 flushed between steps."""
    import torch
    import bit_quantized_mixture_nf4_b200 as e4b
    _, bf16, _, src = peaks()
    layer = Layer(w, dev, path=e4b.PATH_GROUPED, act=e4b.ACT_CLAMPED_GLU, biases=True)
    ms, kernels, _ = timed_steps(layer, steps, 3, flush, torch.cuda.current_stream())
    st = step_stats(ms)
    tf = 12 * w.H * w.I * w.P / (st["median"] / 1e3) / 1e12
    del layer
    torch.cuda.empty_cache()
    return {"workload": workload_desc(w).replace("fwd (", "clamped GLU + per-expert biases, fwd ("),
            "step_ms": st, "tokens_per_s": w.T / (st["median"] / 1e3),
            "roofline": {"bound": "tensor", "achieved": tf, "peak": bf16, "unit": "TFLOP/s", "frac": tf / bf16,
                         "peak_kind": f"{src} bf16 dense (burst)"}}


def router_leg(layer, flush, steps=10):
    """Routing gradient (weights and logits) on the headline layer and batch."""
    import torch
    import bit_quantized_mixture_nf4_b200 as e4b
    _, bf16, _, src = peaks()
    w = layer.w
    dev = layer.dev
    dwt = torch.empty(w.T, w.k, dtype=torch.float32, device=dev)
    dlg = torch.empty(w.T, w.E, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def rstep():
        e4b.e4b_moe_backward_router(layer.desc, layer.experts, layer.x, layer.idx, layer.wts, layer.go,
                                    router_logits=layer.logits, grad_topk_w=dwt, grad_logits=dlg, ws=layer.ws,
                                    stream=stream)

    for _ in range(3):
        rstep()
    torch.cuda.synchronize()
    ms = []
    for _ in range(steps):
        flush.zero_()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        rstep()
        e.record(stream)
        torch.cuda.synchronize()
        ms.append(s.elapsed_time(e))
    st = step_stats(ms)
    r_flops = 6 * w.H * w.I * w.P
    tf = r_flops / (st["median"] / 1e3) / 1e12
    return {"workload": f"same layer and batch as the headline step (T={w.T})", "ms": st,
            "roofline": {"bound": "tensor", "achieved": tf, "peak": bf16, "unit": "TFLOP/s", "frac": tf / bf16,
                         "peak_kind": f"{src} bf16 dense (burst)"},
            "work": "h and the unweighted expert outputs recomputed by the grouped GEMMs (6*H*I FLOP per pair), "
                    "then one fp32 dot product per pair and the softmax backward per token"}


def router_fused_leg(layer, flush, steps=10):
    """The training step with the routing gradient (grad_topk_w and grad_logits)
    fused into the input gradient, against the same step without it.  The extra
    work is one dot product per pair over I, fed from the down^T GEMM's
    accumulator and the saved h, plus the per-token softmax backward; its
    algorithmic bytes: h read (2I B per pair), the per-tile partials written and
    read (8 B per pair and 256-column tile), the routing gradient written (4 B per
    pair), the logits read and their gradient written (8E B per token)."""
    import torch
    hbm = peaks()[0]
    w = layer.w
    stream = torch.cuda.current_stream()
    ms0, _, _ = timed_steps(layer, steps, 3, flush, stream, kinds=())
    layer.with_routing_gradient()
    ms1, _, _ = timed_steps(layer, steps, 3, flush, stream, kinds=())
    layer.routing = False
    s0, s1 = step_stats(ms0), step_stats(ms1)
    nt = -(-w.I // 256)
    extra_bytes = w.P * (2 * w.I + 8 * nt + 4) + w.T * 8 * w.E
    added_ms = s1["median"] - s0["median"]
    roof = None
    if added_ms > 0:
        gbs = extra_bytes / (added_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                "basis": "extra algorithmic bytes / added step time"}
    return {"workload": f"same layer and batch as the headline step (T={w.T})",
            "step_ms_without": s0, "step_ms_with": s1, "added_frac": added_ms / s0["median"],
            "extra_bytes_per_step": extra_bytes, "roofline": roof,
            "work": "forward saves h; e4b_moe_backward: the down^T GEMM epilogue leaves <grad_out W_d, h> per "
                    "row and 256-column tile, a per-token kernel sums them and runs the softmax backward"}


def storage_leg(w, dev, flush, steps=10):
    """The fwd+dgrad step of workload w in every storage format: the 4-bit
    codebooks NF4 / FP4, native MXFP4, the 8-bit blockwise int8 / fp8 (dequantized
    to bf16 one stack at a time before each GEMM) and bf16 passthrough."""
    import torch
    from bit_quantized_mixture_nf4_b200 import workloads as wl
    _, bf16, _, src = peaks()
    out = {"workload": workload_desc(w)}
    for name, cb in (("nf4", wl.NF4), ("fp4", wl.FP4), ("mxfp4", wl.MXFP4), ("int8", wl.INT8), ("fp8", wl.FP8),
                     ("bf16", wl.BF16_WEIGHTS)):
        layer = Layer(dataclasses.replace(w, codebook=cb), dev)
        ms, _, _ = timed_steps(layer, steps, 3, flush, torch.cuda.current_stream(), kinds=())
        del layer
        torch.cuda.empty_cache()
        st = step_stats(ms)
        tf = 12 * w.H * w.I * w.P / (st["median"] / 1e3) / 1e12
        out[name] = {"step_ms": st, "tokens_per_s": w.T / (st["median"] / 1e3), "frac": tf / bf16}
    out["peak_kind"] = f"{src} bf16 dense (burst)"
    return out


def lora_leg(w, dev, flush, rank=16, steps=10):
    """The training step with per-expert LoRA adapters of rank r on both stacks:
    forward (saving g/u and h) + the one-pass backward with the input gradient and
    the four adapter gradients, against the same step of the base layer alone."""
    import torch
    _, bf16, _, src = peaks()
    stream = torch.cuda.current_stream()
    base = Layer(w, dev)
    ms0, _, _ = timed_steps(base, steps, 3, flush, stream, kinds=())
    del base
    torch.cuda.empty_cache()
    layer = Layer(w, dev, lora_rank=rank)
    layer.saved_h = torch.empty(w.P, w.I, dtype=torch.bfloat16, device=dev)
    ms1, _, _ = timed_steps(layer, steps, 3, flush, stream, kinds=())
    del layer
    torch.cuda.empty_cache()
    s0, s1 = step_stats(ms0), step_stats(ms1)
    base_flops = 12 * w.H * w.I * w.P
    # adapter work: the extra 64-deep k-stage in the four GEMMs (rank padded to 64), the
    # four thin projections and the four adapter gradients (2 FLOP per multiply-add)
    k64 = 2 * w.P * 64 * (2 * w.I + w.H + w.I + w.H)
    thin = 2 * w.P * rank * (w.H + w.I + w.H + 2 * w.I)
    grads = 2 * w.P * rank * (w.H + w.I + 2 * w.I + w.H)
    tf = base_flops / (s1["median"] / 1e3) / 1e12
    return {"workload": workload_desc(w).replace("+ dgrad", f"+ dgrad, LoRA r={rank} on both stacks"),
            "step_ms_base": s0, "step_ms_lora": s1, "added_frac": s1["median"] / s0["median"] - 1.0,
            "tokens_per_s": w.T / (s1["median"] / 1e3), "adapter_flops_per_step": k64 + thin + grads,
            "roofline": {"bound": "tensor", "achieved": tf, "peak": bf16, "unit": "TFLOP/s", "frac": tf / bf16,
                         "basis": "base-layer FLOP (12 H I per pair) / LoRA step time",
                         "peak_kind": f"{src} bf16 dense (burst)"}}


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
    res["workload"] = f"{w.name}-shaped gate_up stack [{w.E},{2 * w.I},{w.H}] {('nf4', 'fp4', 'mxfp4', 'int8', 'fp8', 'bf16')[w.codebook]}"
    del gu, out
    torch.cuda.empty_cache()
    return res


def reconstruction_leg(w, dev):
    """NF4 vs FP4 reconstruction error of the same seeded N(0, 0.02) stacks (the
    gpt-oss-shaped layer): relative RMSE ||w - deq(q(w))|| / ||w|| of the bf16
    dequantized weights, quantized and dequantized by the library."""
    import torch
    import bit_quantized_mixture_nf4_b200 as e4b
    from bit_quantized_mixture_nf4_b200 import workloads as wl
    gu, dn = wl.weights(w, device=dev)
    res = {"workload": f"{w.name}-shaped stacks gate_up [{w.E},{2 * w.I},{w.H}] + down [{w.E},{w.H},{w.I}], "
                       f"N(0, 0.02)"}
    for name, cb in (("nf4", e4b.NF4), ("fp4", e4b.FP4)):
        num = den = 0.0
        for stack in (gu, dn):
            p, a = e4b.e4b_quantize_nf4(stack, codebook=cb)
            d = e4b.e4b_dequantize_nf4(p, a, tuple(stack.shape), codebook=cb, out_dtype=e4b.BF16)
            num += float((stack - d.float()).double().pow(2).sum())
            den += float(stack.double().pow(2).sum())
            del p, a, d
        res[f"{name}_rel_rmse"] = (num / den) ** 0.5
    num = den = 0.0
    for stack in (gu, dn):   # native MXFP4 (32-element blocks, E8M0 scales)
        p, sc = e4b.e4b_quantize_mxfp4(stack)
        d = e4b.e4b_dequantize_mxfp4(p, sc, tuple(stack.shape))
        num += float((stack - d.float()).double().pow(2).sum())
        den += float(stack.double().pow(2).sum())
        del p, sc, d
    res["mxfp4_rel_rmse"] = (num / den) ** 0.5
    del gu, dn
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------------ CPU oracle

class OracleSample:
    """The CPU oracle on a bounded sample of a workload.

    One step of the oracle = routing and grouping of all T tokens, dequantization
    of both weight stacks, forward + input gradient of all T tokens.  Routing and
    grouping run in full; dequantization is timed on a fixed sample of blocks and
    scaled to the whole stacks; forward + input gradient are timed on S sampled
    tokens (chosen among the tokens whose experts lie in a subset X whose
    dequantized weights fit a bounded host budget) and scaled linearly to T."""

    MAX_X_ELEMENTS = 400_000_000
    DEQ_SAMPLE = 1 << 24

    def __init__(self, w, seed=0):
        import numpy as np
        import oracle
        from bit_quantized_mixture_nf4_b200 import workloads as wl
        self.w = w
        self.cores = oracle.num_threads()
        x = wl.activations(w)
        self.x = x.float().numpy()
        self.logits = wl.router_logits(w, x).numpy()
        self.go = wl.grad_output(w).float().numpy()
        gu, dn = wl.weights(w)
        self.pg, self.ag = oracle.quantize(gu.numpy(), w.codebook)
        self.pd, self.ad = oracle.quantize(dn.numpy(), w.codebook)
        del gu, dn
        self.idx, self.wts = oracle.route(self.logits, w.k, w.renorm)
        per_expert = 3 * w.H * w.I
        rng = np.random.default_rng(seed)
        X, toks = set(), []
        for t in rng.permutation(w.T):
            ex = set(int(e) for e in self.idx[t])
            if (len(X | ex)) * per_expert <= max(self.MAX_X_ELEMENTS, w.k * per_expert):
                X |= ex
                toks.append(int(t))
        self.X = np.array(sorted(X), np.int64)
        self.pool = np.array(toks, np.int64)
        remap = np.full(w.E, -1, np.int32)
        remap[self.X] = np.arange(len(self.X), dtype=np.int32)
        self.sub_idx = remap[self.idx]
        xs = self.X
        self.wgu = oracle.dequantize(self.pg[xs], self.ag[xs], (len(xs), 2 * w.I, w.H), w.codebook)
        self.wd = oracle.dequantize(self.pd[xs], self.ad[xs], (len(xs), w.H, w.I), w.codebook)

    def step(self, S):
        """Seconds of one extrapolated oracle step; S = sampled tokens."""
        import numpy as np
        import oracle
        w = self.w
        t0 = time.perf_counter()
        idx, _ = oracle.route(self.logits, w.k, w.renorm)
        oracle.permute(idx, w.E)
        t1 = time.perf_counter()
        rows = self.deq_rows()
        oracle.dequantize(self.pg[0][: rows * w.H // 2], self.ag[0][: rows * w.H // 64], (1, rows, w.H), w.codebook)
        t2 = time.perf_counter()
        total = w.E * 3 * w.H * w.I
        toks = self.pool[:min(S, len(self.pool))]
        oracle.forward(self.x[toks], self.sub_idx[toks], self.wts[toks], self.wgu, self.wd)
        oracle.dgrad(self.x[toks], self.go[toks], self.sub_idx[toks], self.wts[toks], self.wgu, self.wd)
        t3 = time.perf_counter()
        parts = {"route_s": t1 - t0, "deq_s": (t2 - t1) * total / (rows * w.H), "tok_s": t3 - t2,
                 "sampled_s": t3 - t0}
        return parts["route_s"] + parts["deq_s"] + parts["tok_s"] * w.T / len(toks), len(toks), parts

    def deq_rows(self):
        """Rows of expert 0's gate_up stack in the dequantization sample."""
        return min(self.DEQ_SAMPLE, self.pg.shape[1] * 2) // self.w.H

    def sample_text(self, S):
        w = self.w
        return (f"routing + grouping of all {w.T} tokens; dequantization timed on {self.deq_rows() * w.H} elements and "
                f"scaled to both stacks ({w.E * 3 * w.H * w.I} elements); fwd+dgrad timed on {S} of {w.T} tokens "
                f"(tokens routed within {len(self.X)} of {w.E} experts) and scaled linearly in tokens")


def cpu_rate(w, target_s=15.0):
    """Oracle throughput in routed tokens/s on a bounded sample (one extrapolated step)."""
    o = OracleSample(w)
    _, used, parts = o.step(o.cores)                   # calibration: per-token cost
    per_tok = parts["tok_s"] / used
    S = int((target_s - parts["route_s"] - parts["sampled_s"] + parts["tok_s"]) / max(per_tok, 1e-9))
    S = max(o.cores, min(len(o.pool), (S // o.cores) * o.cores))
    step, used, _ = o.step(S)
    return w.T / step, dict(cores=o.cores, sample=o.sample_text(used))


def run_reference(args, w):
    """The reference arm: the CPU oracle as it stands, on the host cores.  Each
    step runs the bounded sample of OracleSample (8 sampled tokens per core);
    value = T / the extrapolated full step, ms_per_step = the sampled step's own
    wall time."""
    world, rank, _ = dist_env()
    if rank != 0:
        return
    o = OracleSample(w, seed=1)
    S = 8 * o.cores
    used = S
    for _ in range(args.warmup):
        _, used, _ = o.step(S)
    full, wall = [], []
    for _ in range(args.steps):
        s, used, parts = o.step(S)
        full.append(s)
        wall.append(parts["sampled_s"])
    step = statistics.median(full)
    value = w.T / step
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.median(wall) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": bench_config(w, world),
            "extrapolated_full_step_ms": step_stats([s * 1e3 for s in full]),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": o.cores, "kind": "oracle",
                             "sample": o.sample_text(used)},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm

def e2e_leg(layer, steps, world, stream):
    """The same step end to end through the C-ABI's pipelined host-buffer runner:
    every step copies its inputs in from pinned host memory and its y and grad_x
    out, on copy streams that overlap one batch's copies with the neighbouring
    batches' kernels.  The L2 is not flushed: the copies stream ~0.5 GB per step."""
    import torch
    import bit_quantized_mixture_nf4_b200 as e4b
    w = layer.w
    T = w.T
    x_p = layer.x_h.pin_memory()
    l_p = layer.logits_h.pin_memory()
    g_p = layer.go_h.pin_memory()
    y_p = torch.empty(T, w.H, dtype=torch.bfloat16).pin_memory()
    gx_p = torch.empty(T, w.H, dtype=torch.bfloat16).pin_memory()
    pipe = e4b.e4b_pipe_create(layer.desc, layer.experts, T, layer.dev, stream)
    try:
        for _ in range(3):
            e4b.e4b_pipe_submit(pipe, x_p, l_p, g_p, y_p, gx_p)
        e4b.e4b_pipe_sync(pipe)
        if world > 1:
            torch.distributed.barrier()
        es, ee = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        es.record(stream)
        e4b.e4b_pipe_join(pipe)          # the pipe's copies start after es
        for _ in range(steps):
            e4b.e4b_pipe_submit(pipe, x_p, l_p, g_p, y_p, gx_p)
        e4b.e4b_pipe_join(pipe)          # ee after the last copy out
        ee.record(stream)
        e4b.e4b_pipe_sync(pipe)
        torch.cuda.synchronize()
    finally:
        e4b.e4b_pipe_destroy(pipe)
    e2e_ms = max_over_ranks(es.elapsed_time(ee) / steps, layer.dev)
    h2d = x_p.numel() * 2 + l_p.numel() * 4 + g_p.numel() * 2
    d2h = y_p.numel() * 2 + gx_p.numel() * 2
    return {"value": job_throughput(T, world, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
            "api": "e4b_pipe_submit (pinned host buffers; copies of one batch overlap the kernels of the "
                   "neighbouring batches)"}


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
    hbm, bf16_burst, bf16_sus, peak_src = peaks()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)   # > 126 MB L2
    stream = torch.cuda.current_stream()
    layer = Layer(w, dev)

    # ------------------------------------------------ device-timed region
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        step_ms, kernels, launches = timed_steps(layer, args.steps, args.warmup, flush, stream, clk)
    if world > 1:
        torch.distributed.barrier()
    total_ms = max_over_ranks(sum(step_ms), dev)
    ms_per_step = total_ms / args.steps
    value = job_throughput(w.T, world, ms_per_step)
    peak, peak_kind = roofline_peak(total_ms, bf16_burst, bf16_sus, peak_src)
    roof, per_kernel = gemm_roofline(w, kernels, peak, peak_kind, bf16_burst)
    roof["traffic"] = recorded_traffic(roof["kernel"], f"{w.name}_T{w.T}")
    step_tf = 12 * w.H * w.I * w.P / (ms_per_step / 1e3) / 1e12

    # per-kernel breakdown of the rest of the step: a short separate pass with every
    # kind bracketed by events (which serialises the chained small kernels)
    e4b.e4b_timing_reset()
    e4b.e4b_timing_enable(True)
    for _ in range(3):
        flush.zero_()
        layer.step(stream)
    torch.cuda.synchronize()
    e4b.e4b_timing_enable(False)
    small_kernels = {}
    for name in ("route", "group", "gather", "combine"):
        t, n = e4b.e4b_timing_get(name)
        if n:
            small_kernels[name] = {"launches": n, "avg_ms": t / n}

    e2e = None if args.no_e2e else e2e_leg(layer, args.steps, world, stream)

    aux = {}
    if not args.no_aux:
        aux["router_backward"] = router_leg(layer, flush)
        aux["router_fused"] = router_fused_leg(layer, flush)
    del layer
    torch.cuda.empty_cache()
    if not args.no_aux:
        legs = {}
        for v in (wl.OLMOE, wl.QWEN3, wl.GPTOSS, wl.MIXTRAL):
            if v.name != w.name:
                legs[f"{v.name}_T{v.T}"] = step_leg(v, dev, flush)
        aux["large_layers"] = legs
        aux["lora"] = lora_leg(wl.OLMOE, dev, flush)
        aux["storage_formats"] = storage_leg(wl.OLMOE, dev, flush)
        aux["decode"] = [decode_leg(v, dev) for v in (wl.QWEN3.with_tokens(1), wl.QWEN3.with_tokens(2),
                                                      wl.QWEN3.with_tokens(4), wl.QWEN3.with_tokens(8),
                                                      wl.GPTOSS.with_tokens(1))]
        torch.cuda.empty_cache()
        aux["codec"] = codec_leg(wl.OLMOE, dev)
        aux["reconstruction_nf4_vs_fp4"] = reconstruction_leg(wl.GPTOSS, dev)
        aux["gptoss_variant"] = variant_leg(wl.GPTOSS.with_tokens(2048), dev, flush)
        aux["gptoss_variant_mxfp4"] = variant_leg(dataclasses.replace(wl.GPTOSS.with_tokens(2048),
                                                                      codebook=wl.MXFP4), dev, flush)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, info = cpu_rate(w)
        cpu = {"value": rate, "unit": UNIT, "cores": info["cores"], "kind": "oracle", "sample": info["sample"]}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": bench_config(w, world),
            "step_ms": step_stats(step_ms),
            "roofline": roof,
            "step_roofline": {"bound": "tensor", "achieved": step_tf, "peak": peak, "unit": "TFLOP/s",
                              "frac": step_tf / peak, "flops_per_step": 12 * w.H * w.I * w.P,
                              "peak_kind": peak_kind, "frac_of_burst": step_tf / bf16_burst},
            "kernels": per_kernel,
            "small_kernels": {"timed": "separate 3-step pass, every launch bracketed by events", **small_kernels},
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
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
        if args.leg == "decode":
            tokens = args.tokens if 0 < args.tokens <= 8 else 1
            base = wl.QWEN3 if args.workload == "mixtral" else wl.ALL[args.workload]   # decode: Qwen3 by default
            print(json.dumps(decode_leg(base.with_tokens(tokens), dev, reps=max(args.steps, 3))), flush=True)
        elif args.leg == "storage":
            w = headline_workload(args) if args.workload != "mixtral" else wl.OLMOE
            print(json.dumps(storage_leg(w, dev, flush, steps=max(args.steps, 3))), flush=True)
        elif args.leg == "lora":
            w = headline_workload(args)
            print(json.dumps(lora_leg(w, dev, flush, steps=max(args.steps, 3))), flush=True)
        elif args.leg == "router":
            w = headline_workload(args)
            layer = Layer(w, dev)
            print(json.dumps({"router_fused": router_fused_leg(layer, flush, steps=max(args.steps, 3)),
                              "router_backward": router_leg(layer, flush, steps=max(args.steps, 3))}), flush=True)
        elif args.leg == "variant":
            vw = wl.GPTOSS.with_tokens(2048)
            if args.codebook == "mxfp4":
                vw = dataclasses.replace(vw, codebook=wl.MXFP4)
            print(json.dumps(variant_leg(vw, dev, flush, steps=max(args.steps, 3))),
                  flush=True)
        else:
            print(json.dumps(codec_leg(wl.OLMOE, dev, reps=max(args.steps, 3))), flush=True)
        return
    w = headline_workload(args)
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_e4b(args, w)


if __name__ == "__main__":
    main()
