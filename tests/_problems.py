"""Problem construction shared by the tests: seeded inputs from the workload
module, quantized by the ORACLE (so no oracle input ever comes from the CUDA
path), plus oracle references."""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

import oracle
from bit_quantized_mixture_nf4_b200 import workloads as wl


@dataclasses.dataclass
class Problem:
    w: wl.Workload
    x: torch.Tensor            # bf16 [T, H] (CPU)
    logits: torch.Tensor       # fp32 [T, E] (CPU)
    grad_out: torch.Tensor     # bf16 [T, H] (CPU)
    gu: np.ndarray             # fp32 [E, 2I, H]
    dn: np.ndarray             # fp32 [E, H, I]
    pg: np.ndarray             # oracle packed gate_up
    ag: np.ndarray
    pd: np.ndarray             # oracle packed down
    ad: np.ndarray


def custom(name="custom", E=4, H=320, I=192, k=2, renorm=True, T=500, seed=7, codebook=wl.NF4, router="linear",
           router_std=None):
    return wl.Workload(name, E=E, H=H, I=I, k=k, renorm=renorm, T=T, seed=seed, codebook=codebook, router=router,
                       router_std=router_std if router_std is not None else 1.0 / np.sqrt(H))


_cache = {}


def build(w: wl.Workload) -> Problem:
    key = dataclasses.astuple(w)
    if key in _cache:
        return _cache[key]
    x = wl.activations(w)
    gu, dn = wl.weights(w)
    logits = wl.router_logits(w, x)
    go = wl.grad_output(w)
    gu = gu.numpy()
    dn = dn.numpy()
    if w.codebook == wl.MXFP4:   # packed codes + E8M0 scale bytes (in ag / ad)
        pg, ag = oracle.quantize_mxfp4(gu)
        pd, ad = oracle.quantize_mxfp4(dn)
    elif w.codebook in (wl.INT8, wl.FP8):   # one code byte per element
        pg, ag = oracle.quantize8(gu, w.codebook)
        pd, ad = oracle.quantize8(dn, w.codebook)
    elif w.codebook == wl.BF16_WEIGHTS:   # passthrough: the bf16 bits of the weights, no absmax
        pg = torch.from_numpy(gu).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint8)
        pd = torch.from_numpy(dn).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint8)
        ag = ad = np.zeros((w.E, 1), np.float32)
    else:
        pg, ag = oracle.quantize(gu, w.codebook)
        pd, ad = oracle.quantize(dn, w.codebook)
    prob = Problem(w, x, logits, go, gu, dn, pg, ag, pd, ad)
    if len(_cache) > 2:
        _cache.clear()
    _cache[key] = prob
    return prob


def oracle_weights(prob: Problem, experts=None):
    """bf16-dequantized weights (as fp32) of all experts or of a subset (in that order)."""
    w = prob.w
    if experts is None:
        experts = np.arange(w.E)
    experts = np.asarray(experts)
    if w.codebook == wl.MXFP4:
        wgu = oracle.dequantize_mxfp4(prob.pg[experts], prob.ag[experts], (len(experts), 2 * w.I, w.H))
        wd = oracle.dequantize_mxfp4(prob.pd[experts], prob.ad[experts], (len(experts), w.H, w.I))
        return wgu, wd
    if w.codebook in (wl.INT8, wl.FP8):
        wgu = oracle.dequantize8(prob.pg[experts], prob.ag[experts], (len(experts), 2 * w.I, w.H), w.codebook)
        wd = oracle.dequantize8(prob.pd[experts], prob.ad[experts], (len(experts), w.H, w.I), w.codebook)
        return wgu, wd
    if w.codebook == wl.BF16_WEIGHTS:
        bits = lambda a, shape: oracle.bf16_bits_to_f32(np.ascontiguousarray(a).view(np.uint16).reshape(shape))
        return (bits(prob.pg[experts], (len(experts), 2 * w.I, w.H)), bits(prob.pd[experts], (len(experts), w.H, w.I)))
    wgu = oracle.dequantize(prob.pg[experts], prob.ag[experts], (len(experts), 2 * w.I, w.H), w.codebook)
    wd = oracle.dequantize(prob.pd[experts], prob.ad[experts], (len(experts), w.H, w.I), w.codebook)
    return wgu, wd


def oracle_forward_dgrad(prob: Problem, idx: np.ndarray, wts: np.ndarray, tokens, want_dgrad=True, act=0,
                         alpha=1.702, limit=7.0, bgu=None, bd=None):
    """Oracle y (and grad_x) for the given tokens, using only the experts they touch;
    act / alpha / limit and the per-expert biases bgu [E, 2I], bd [E, H] as in the
    oracle's forward."""
    tokens = np.asarray(tokens, np.int64)
    used = np.unique(idx[tokens])
    remap = np.full(prob.w.E, -1, np.int32)
    remap[used] = np.arange(len(used), dtype=np.int32)
    wgu, wd = oracle_weights(prob, used)
    sub_idx = remap[idx[tokens]]
    sub_w = wts[tokens]
    xs = prob.x.float().numpy()[tokens]
    kw = dict(act=act, alpha=alpha, limit=limit, bgu=None if bgu is None else np.asarray(bgu)[used])
    y = oracle.forward(xs, sub_idx, sub_w, wgu, wd, bd=None if bd is None else np.asarray(bd)[used], **kw)
    gx = None
    if want_dgrad:
        gos = prob.grad_out.float().numpy()[tokens]
        gx = oracle.dgrad(xs, gos, sub_idx, sub_w, wgu, wd, **kw)
    return y, gx


def to_dev(a, device="cuda"):
    if isinstance(a, np.ndarray):
        a = torch.from_numpy(np.ascontiguousarray(a))
    return a.to(device).contiguous()


def assert_close_rel_max(got: np.ndarray, ref: np.ndarray, rel=1e-2, what=""):
    """max|got - ref| <= rel * max|ref| (the forward / dgrad tolerance)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = np.abs(ref).max()
    err = np.abs(got - ref).max()
    assert err <= rel * scale, f"{what}: max|diff| {err:.3e} > {rel} * max|ref| {scale:.3e}"
    return err / scale
