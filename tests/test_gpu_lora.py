"""Per-expert LoRA over the frozen 4-bit base ("experts4bit-qlora" 0.4.0
description, "ExpertsLoRA(base, r, alpha)": only the adapters train) through the
C ABI, against the oracle's lora_forward / lora_backward (fp64): the forward
output, the input gradient and the four adapter gradients within
max|diff| <= 1e-2 * max|ref|.  Pins besides the oracle: zero B adapters give
the base forward bit for bit, and the saved and recompute backward modes agree
bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_mixture_nf4_b200 import workloads as wl
from tests import _problems as pb
from tests.test_gpu_parity import _check_status

pytestmark = pytest.mark.gpu

TOL = 1e-2


@pytest.fixture(scope="module")
def e4b():
    import bit_quantized_mixture_nf4_b200 as m
    m.lib
    return m


def _adapters(w, r, seed, zero_b=False):
    """bf16-representable adapters (A ~ N(0, 1/in), B ~ N(0, 0.01/r)) as fp32 numpy."""
    rng = np.random.default_rng(seed)
    def bf(a):
        return torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16).float().numpy()
    agu = bf(rng.standard_normal((w.E, r, w.H)) / np.sqrt(w.H))
    bgu = bf(rng.standard_normal((w.E, 2 * w.I, r)) * 0.1 / np.sqrt(r)) * (0.0 if zero_b else 1.0)
    ad = bf(rng.standard_normal((w.E, r, w.I)) / np.sqrt(w.I))
    bd = bf(rng.standard_normal((w.E, w.H, r)) * 0.1 / np.sqrt(r)) * (0.0 if zero_b else 1.0)
    return agu, bgu, ad, bd


def _layer(e4b, prob, r, scale, lora_np, act=0, limit=7.0, biases=None):
    w = prob.w
    t = {k: pb.to_dev(getattr(prob, k)) for k in ("pg", "ag", "pd", "ad")}
    lt = None if lora_np is None else tuple(torch.from_numpy(a).to(torch.bfloat16).cuda() for a in lora_np)
    bt = None if biases is None else tuple(pb.to_dev(b) for b in biases)
    experts = e4b.make_experts(t["pg"], t["pd"], t["ag"], t["ad"], *(bt or (None, None)), lora=lt)
    d = e4b.make_desc(w.E, w.H, w.I, w.k, w.renorm, w.codebook, 64, e4b.PATH_GROUPED, act, 1.702, limit,
                      lora_rank=r if lora_np is not None else 0, lora_scale=scale)
    return d, experts, (t, lt, bt)


def _run(e4b, w, r, scale, act=0, limit=7.0, with_biases=False, seed=0):
    prob = pb.build(w)
    lora = _adapters(w, r, 90 + seed)
    biases = None
    if with_biases:
        from tests.test_gpu_variant import _biases
        biases = _biases(w, 91 + seed)
    d, experts, keep = _layer(e4b, prob, r, scale, lora, act, limit, biases)
    x = pb.to_dev(prob.x)
    logits = pb.to_dev(prob.logits)
    go = pb.to_dev(prob.grad_out)
    P = w.T * w.k
    sgu = torch.empty(P, 2 * w.I, dtype=torch.bfloat16, device="cuda")
    sh = torch.empty(P, w.I, dtype=torch.bfloat16, device="cuda")
    y, idx, wts = e4b.e4b_moe_forward(d, experts, x, logits, saved_gu=sgu, saved_h=sh)
    grads = tuple(torch.empty(a.shape, dtype=torch.float32, device="cuda") for a in lora)
    gx, dw, dl = e4b.e4b_moe_backward(d, experts, x, idx, wts, go, saved_gu=sgu, saved_h=sh, router_logits=logits,
                                      lora_grads=grads)
    grads_re = tuple(torch.empty_like(g) for g in grads)
    gx_re, dw_re, _ = e4b.e4b_moe_backward(d, experts, x, idx, wts, go, router_logits=logits, lora_grads=grads_re)
    gx_sep = e4b.e4b_moe_backward_dgrad(d, experts, None, idx, wts, go, saved_gu=sgu)   # grad_x only, no x
    torch.cuda.synchronize()
    _check_status(e4b)
    assert torch.equal(gx, gx_re) and torch.equal(dw, dw_re) and torch.equal(gx, gx_sep)
    for g, g2 in zip(grads, grads_re):
        assert torch.equal(g, g2)
    gi = idx.cpu().numpy()
    oi, ow = oracle.route(prob.logits.numpy(), w.k, w.renorm)
    assert np.array_equal(gi, oi)
    wgu, wdn = pb.oracle_weights(prob)
    bgu, bd = biases if biases is not None else (None, None)
    ow64 = wts.cpu().numpy().astype(np.float64)
    yref = oracle.lora_forward(prob.x.float().numpy(), gi, ow64, wgu, wdn, *lora, scale, act=act, limit=limit,
                               bgu=bgu, bd=bd)
    pb.assert_close_rel_max(y.float().cpu().numpy(), yref, TOL, "LoRA forward")
    gref = oracle.lora_backward(prob.x.float().numpy(), prob.grad_out.float().numpy(), gi, ow64, wgu, wdn, *lora,
                                scale, act=act, limit=limit, bgu=bgu)
    pb.assert_close_rel_max(gx.float().cpu().numpy(), gref[0], TOL, "LoRA grad_x")
    for name, g, ref in zip(("dA_gu", "dB_gu", "dA_d", "dB_d"), grads, gref[1:]):
        pb.assert_close_rel_max(g.cpu().numpy(), ref, TOL, f"LoRA {name}")
    return prob, keep


@pytest.mark.parametrize("w,r", [
    (pb.custom("lora_a", E=4, H=256, I=192, k=2, T=100, seed=81), 8),      # I not a multiple of 128
    (pb.custom("lora_b", E=6, H=320, I=256, k=2, T=150, seed=82), 16),
    (pb.custom("lora_fp4", E=4, H=256, I=384, k=2, T=90, seed=83, codebook=wl.FP4), 64),
], ids=["r8", "r16", "r64-fp4"])
def test_lora_forward_backward_matches_oracle(e4b, w, r):
    _run(e4b, w, r, scale=2.0)


def test_lora_with_variant(e4b):
    """Adapters on the clamped-GLU experts (gpt-oss alpha 1.702, limit 7) with
    per-expert biases.  A tight limit is left to the variant tests: there the
    clamp's derivative mask flips on pre-activations within rounding of the limit,
    and the adapter term moves that rounding."""
    w = pb.custom("lora_v", E=4, H=256, I=192, k=2, T=80, seed=84)
    _run(e4b, w, 16, scale=1.5, act=1, limit=7.0, with_biases=True, seed=1)


def test_lora_olmoe_shaped(e4b):
    """OLMoE-shaped layer (E=64, H=2048, I=1024, top-8) at T=32 with r=16."""
    _run(e4b, wl.OLMOE.with_tokens(32), 16, scale=1.0, seed=2)


def test_lora_zero_b_is_the_base(e4b):
    """B adapters = 0: the forward and the input gradient equal the base layer's
    bit for bit (the extra k-stage adds exact zeros)."""
    w = pb.custom("lora_z", E=4, H=256, I=192, k=2, T=64, seed=85)
    prob = pb.build(w)
    lora = _adapters(w, 16, 92, zero_b=True)
    d, experts, keep = _layer(e4b, prob, 16, 2.0, lora)
    d0, experts0, keep0 = _layer(e4b, prob, 0, 1.0, None)
    x = pb.to_dev(prob.x)
    logits = pb.to_dev(prob.logits)
    go = pb.to_dev(prob.grad_out)
    y, idx, wts = e4b.e4b_moe_forward(d, experts, x, logits)
    y0, _, _ = e4b.e4b_moe_forward(d0, experts0, x, logits)
    gx = e4b.e4b_moe_backward_dgrad(d, experts, x, idx, wts, go)
    gx0 = e4b.e4b_moe_backward_dgrad(d0, experts0, x, idx, wts, go)
    torch.cuda.synchronize()
    _check_status(e4b)
    assert torch.equal(y, y0)
    assert torch.equal(gx, gx0)
