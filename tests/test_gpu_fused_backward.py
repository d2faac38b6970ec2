"""The layer backward in one pass (e4b_moe_backward): the input gradient and the
routing gradient, with the routing-weight gradient fused into the input
gradient's down^T GEMM.  Since the routing weight multiplies the expert output
("experts4bit-qlora 0.1.0" source diff, _vendor/experts.py,
Experts4bit.forward), dL/dw_{t,j} = <grad_out_t, Y_{t,j}> = <grad_out_t W_d, h_{t,j}>
(+ <grad_out_t, b_e> with a down bias).  Checked against the oracle's
router_grad (fp64) within max|diff| <= 1e-2 * max|ref|.  grad_x must equal the
separate input-gradient call bit for bit (same kernels), and the saved and
recomputed modes must agree bit for bit (the same gate_up kernel makes h)."""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_mixture_nf4_b200 import workloads as wl
from tests import _problems as pb
from tests.test_gpu_parity import _check_status, _desc, _upload_experts
from tests.test_gpu_router_grad import _oracle_router

pytestmark = pytest.mark.gpu

TOL = 1e-2


@pytest.fixture(scope="module")
def e4b():
    import bit_quantized_mixture_nf4_b200 as m
    m.lib
    return m


def _forward_saved(e4b, w, d, experts, x, logits):
    P = w.T * w.k
    saved_gu = torch.empty(P, 2 * w.I, dtype=torch.bfloat16, device="cuda")
    saved_h = torch.empty(P, w.I, dtype=torch.bfloat16, device="cuda")
    y, idx, wts = e4b.e4b_moe_forward(d, experts, x, logits, saved_gu=saved_gu, saved_h=saved_h)
    return y, idx, wts, saved_gu, saved_h


def _check(e4b, prob, tokens, experts, d, act=0, alpha=1.702, limit=7.0, bgu=None, bd=None):
    w = prob.w
    x = pb.to_dev(prob.x)
    logits = pb.to_dev(prob.logits)
    go = pb.to_dev(prob.grad_out)
    y, idx, wts, sgu, sh = _forward_saved(e4b, w, d, experts, x, logits)
    y0, _, _ = e4b.e4b_moe_forward(d, experts, x, logits)   # saved_h must not change the forward
    gx, dw, dl = e4b.e4b_moe_backward(d, experts, x, idx, wts, go, saved_gu=sgu, saved_h=sh, router_logits=logits)
    gx_sep = e4b.e4b_moe_backward_dgrad(d, experts, x, idx, wts, go, saved_gu=sgu)
    gx_re, dw_re, dl_re = e4b.e4b_moe_backward(d, experts, x, idx, wts, go, router_logits=logits)   # recompute
    _, dw_only, _ = e4b.e4b_moe_backward(d, experts, x, idx, wts, go, saved_gu=sgu, saved_h=sh,
                                         want_grad_x=False)   # routing only, no logits
    torch.cuda.synchronize()
    _check_status(e4b)
    assert torch.equal(y, y0)
    assert torch.equal(gx, gx_sep)
    assert torch.equal(gx, gx_re) and torch.equal(dw, dw_re) and torch.equal(dl, dl_re)
    assert torch.equal(dw, dw_only)
    gi = idx.cpu().numpy()
    assert np.array_equal(gi, oracle.route(prob.logits.numpy(), w.k, w.renorm)[0])
    if bd is None and act == 0 and bgu is None:
        rdw, rdl = _oracle_router(prob, gi, tokens)
    else:
        wgu, wdn = pb.oracle_weights(prob)
        rdw, rdl = oracle.router_grad(prob.x.float().numpy(), prob.grad_out.float().numpy(), prob.logits.numpy(),
                                      gi, w.renorm, wgu, wdn, tokens=tokens, act=act, alpha=alpha, limit=limit,
                                      bgu=bgu, bd=bd)
    pb.assert_close_rel_max(dw.cpu().numpy()[tokens], rdw, TOL, "grad_topk_w (fused)")
    pb.assert_close_rel_max(dl.cpu().numpy()[tokens], rdl, TOL, "grad_logits (fused)")
    return gx, dw, dl


@pytest.mark.parametrize("wname,T", [("tiny", 64), ("olmoe", 40), ("qwen3", 48), ("gptoss", 24)])
def test_fused_backward_matches_oracle(e4b, wname, T):
    w = wl.ALL[wname].with_tokens(T)
    prob = pb.build(w)
    keep, experts = _upload_experts(e4b, prob)   # keep: the device tensors behind experts
    _check(e4b, prob, np.arange(T), experts, _desc(e4b, w, e4b.PATH_GROUPED))


@pytest.mark.parametrize("act,limit", [(1, 0.8), (0, 7.0)], ids=["clamped_glu", "swiglu"])
def test_fused_backward_with_biases(e4b, act, limit):
    """Per-expert biases: the down bias adds <grad_out_t, b_e> to dw."""
    from tests.test_gpu_variant import _biases
    w = pb.custom("fb_bias", E=8, H=256, I=448, k=2, T=150, seed=57)   # I = 448: a partial 256-column tile
    prob = pb.build(w)
    bgu, bd = _biases(w, 58)
    t = {k: pb.to_dev(getattr(prob, k)) for k in ("pg", "ag", "pd", "ad")}
    tb, td = pb.to_dev(bgu), pb.to_dev(bd)   # kept alive: the descriptor holds raw pointers
    experts = e4b.make_experts(t["pg"], t["pd"], t["ag"], t["ad"], tb, td)
    d = e4b.make_desc(w.E, w.H, w.I, w.k, w.renorm, w.codebook, 64, e4b.PATH_GROUPED, act, 1.702, limit)
    _check(e4b, prob, np.arange(w.T), experts, d, act=act, limit=limit, bgu=bgu, bd=bd)
    del t, tb, td


def test_fused_backward_full_size_sampled(e4b):
    """The OLMoE-shaped layer at T=4096 in the launch configuration the bench
    times: dw and dlogits on sampled tokens, and dw of every pair against the
    separate (recompute) routing-gradient call."""
    w = wl.OLMOE
    prob = pb.build(w)
    keep, experts = _upload_experts(e4b, prob)   # keep: the device tensors behind experts
    d = _desc(e4b, w, e4b.PATH_GROUPED)
    toks = np.random.default_rng(4).choice(w.T, size=12, replace=False)
    gx, dw, dl = _check(e4b, prob, toks, experts, d)
    x = pb.to_dev(prob.x)
    logits = pb.to_dev(prob.logits)
    _, idx2, wts = e4b.e4b_moe_forward(d, experts, x, logits)
    dw_sep, dl_sep = e4b.e4b_moe_backward_router(d, experts, x, idx2, wts, pb.to_dev(prob.grad_out),
                                                 router_logits=logits)
    torch.cuda.synchronize()
    # the separate call rounds Y to bf16 per row; the fused one takes <grad_out W_d, h> in fp32
    scale = float(dw_sep.abs().max())
    assert float((dw - dw_sep).abs().max()) <= TOL * scale
