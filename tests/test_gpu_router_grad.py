"""Routing gradient (e4b_moe_backward_router) against the oracle: the gradient of
L = <grad_out, y> with respect to the routing weights and the router logits,
indices held.  Tolerance max|diff| <= 1e-2 * max|ref| (the expert outputs pass
through bf16 like every slot row; the oracle is fp64)."""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_mixture_nf4_b200 import workloads as wl
from tests import _problems as pb
from tests.test_gpu_parity import _check_status, _desc, _upload_experts

pytestmark = pytest.mark.gpu

TOL = 1e-2


@pytest.fixture(scope="module")
def e4b():
    import bit_quantized_mixture_nf4_b200 as m
    m.lib
    return m


def _oracle_router(prob, idx, tokens):
    """Oracle dw / dlogits for the given tokens.  Only the experts those tokens
    touch are dequantized; the stacks hold zeros elsewhere (never read)."""
    w = prob.w
    tokens = np.asarray(tokens, np.int64)
    used = np.unique(idx[tokens])
    wgu, wd = pb.oracle_weights(prob, used)
    fg = np.zeros((w.E,) + wgu.shape[1:], np.float32)
    fd = np.zeros((w.E,) + wd.shape[1:], np.float32)
    fg[used] = wgu
    fd[used] = wd
    return oracle.router_grad(prob.x.float().numpy(), prob.grad_out.float().numpy(), prob.logits.numpy(), idx,
                              w.renorm, fg, fd, tokens=tokens)


def _run(e4b, prob, tokens, with_logits=True):
    w = prob.w
    _, experts = _upload_experts(e4b, prob)
    d = _desc(e4b, w, e4b.PATH_GROUPED)
    x = pb.to_dev(prob.x)
    logits = pb.to_dev(prob.logits)
    y, idx, wts = e4b.e4b_moe_forward(d, experts, x, logits)
    go = pb.to_dev(prob.grad_out)
    dw, dl = e4b.e4b_moe_backward_router(d, experts, x, idx, wts, go, router_logits=logits if with_logits else None)
    torch.cuda.synchronize()
    _check_status(e4b)
    gi = idx.cpu().numpy()
    oi, _ = oracle.route(prob.logits.numpy(), w.k, w.renorm)
    assert np.array_equal(gi, oi)
    rdw, rdl = _oracle_router(prob, gi, tokens)
    pb.assert_close_rel_max(dw.cpu().numpy()[tokens], rdw, TOL, "grad_topk_w")
    if with_logits:
        got = dl.cpu().numpy()[tokens]
        pb.assert_close_rel_max(got, rdl, TOL, "grad_logits")
        if w.renorm:   # logits outside the top-k get exactly 0
            for i, t in enumerate(tokens):
                assert np.all(np.delete(got[i], gi[t]) == 0.0)
    else:
        assert dl is None


@pytest.mark.parametrize("wname,T", [("tiny", 64), ("olmoe", 40), ("qwen3", 48), ("gptoss", 24)])
def test_router_grad_matches_oracle(e4b, wname, T):
    w = wl.ALL[wname].with_tokens(T)
    prob = pb.build(w)
    _run(e4b, prob, np.arange(T))


def test_router_grad_without_logits_and_arg_checks(e4b):
    w = pb.custom("rg", E=8, H=256, I=128, k=2, T=33, seed=51)
    prob = pb.build(w)
    _run(e4b, prob, np.arange(w.T), with_logits=False)
    _, experts = _upload_experts(e4b, prob)
    d = _desc(e4b, w, e4b.PATH_GROUPED)
    x = pb.to_dev(prob.x)
    idx = torch.zeros(w.T, w.k, dtype=torch.int32, device="cuda")
    wts = torch.ones(w.T, w.k, dtype=torch.float32, device="cuda")
    go = pb.to_dev(prob.grad_out)
    dl = torch.empty(w.T, w.E, dtype=torch.float32, device="cuda")
    with pytest.raises(e4b.E4BError):   # grad_logits without router_logits
        e4b.e4b_moe_backward_router(d, experts, x, idx, wts, go, router_logits=None, grad_logits=dl)


def test_router_grad_full_size_sampled(e4b):
    """The benchmark's OLMoE-shaped layer at T=4096, checked on sampled tokens."""
    w = wl.OLMOE
    prob = pb.build(w)
    toks = np.random.default_rng(3).choice(w.T, size=12, replace=False)
    _run(e4b, prob, toks)
