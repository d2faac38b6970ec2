"""The gpt-oss expert variant ("experts4bit-qlora 0.31.1" project page, section
"Scope": per-expert biases and a clamped GLU) through the C ABI, against the
oracle: routing exact, forward and input gradient within max|diff| <= 1e-2 *
max|ref|, the routing gradient likewise.  The decode kernels do not implement
the variant: AUTO must take the grouped kernels at T <= 8 and DECODE is refused."""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_mixture_nf4_b200 import workloads as wl
from tests import _problems as pb
from tests.test_gpu_parity import TOL, _check_routing, _check_status, _sample_tokens

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def e4b():
    import bit_quantized_mixture_nf4_b200 as m
    m.lib
    return m


def _biases(w, seed, scale=0.3):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((w.E, 2 * w.I)) * scale).astype(np.float32), \
        (rng.standard_normal((w.E, w.H)) * scale).astype(np.float32)


def _run(e4b, prob, act, alpha, limit, bgu, bd, path=None, T=None, want_dgrad=True):
    w = prob.w
    t = {k: pb.to_dev(getattr(prob, k)) for k in ("pg", "ag", "pd", "ad")}
    tb = None if bgu is None else pb.to_dev(bgu)
    td = None if bd is None else pb.to_dev(bd)
    experts = e4b.make_experts(t["pg"], t["pd"], t["ag"], t["ad"], tb, td)
    d = e4b.make_desc(w.E, w.H, w.I, w.k, w.renorm, w.codebook, 64, e4b.PATH_GROUPED if path is None else path,
                      act, alpha, limit)
    x = pb.to_dev(prob.x)
    lg = pb.to_dev(prob.logits)
    saved = torch.empty(w.T * w.k, 2 * w.I, dtype=torch.bfloat16, device="cuda") if want_dgrad else None
    offs = torch.empty(w.E + 1, dtype=torch.int32, device="cuda") if want_dgrad else None
    perm = torch.empty(w.T * w.k, dtype=torch.int32, device="cuda") if want_dgrad else None
    y, idx, wts = e4b.e4b_moe_forward(d, experts, x, lg, saved_gu=saved, offsets_out=offs, perm_out=perm)
    gx = None
    if want_dgrad:
        go = pb.to_dev(prob.grad_out)
        gx = e4b.e4b_moe_backward_dgrad(d, experts, x, idx, wts, go, saved_gu=saved)
        gx_re = e4b.e4b_moe_backward_dgrad(d, experts, x, idx, wts, go)   # derivatives recomputed from x
        torch.cuda.synchronize()
        assert torch.equal(gx, gx_re)
    torch.cuda.synchronize()
    _check_status(e4b)
    keep = (t, tb, td)   # the device tensors behind `experts`
    return dict(y=y, idx=idx, wts=wts, offs=offs, perm=perm, gx=gx, d=d, experts=experts, x=x, keep=keep)


VARIANTS = [
    # (name, activation, alpha, limit, gate_up bias, down bias)
    ("glu_bias", 1, 1.702, 7.0, True, True),
    ("glu_tight_limit", 1, 1.702, 0.5, True, False),   # the clamp active on many g and u
    ("glu_nobias", 1, 1.0, float("inf"), False, False),
    ("swiglu_bias", 0, 1.702, 7.0, True, True),         # biases with the plain activation
]
SHAPES = [
    pb.custom("v_ragged", E=6, H=320, I=192, k=2, T=400, seed=51),
    pb.custom("v_fp4", E=8, H=256, I=384, k=4, T=300, seed=52, codebook=wl.FP4),
]


@pytest.mark.parametrize("w", SHAPES, ids=lambda w: w.name)
@pytest.mark.parametrize("name,act,alpha,limit,has_bgu,has_bd", VARIANTS, ids=[v[0] for v in VARIANTS])
def test_variant_forward_and_dgrad(e4b, w, name, act, alpha, limit, has_bgu, has_bd):
    prob = pb.build(w)
    bgu, bd = _biases(w, 60 + w.seed)
    bgu = bgu if has_bgu else None
    bd = bd if has_bd else None
    r = _run(e4b, prob, act, alpha, limit, bgu, bd)
    oi, ow = _check_routing(prob, r)
    yref, gref = pb.oracle_forward_dgrad(prob, oi, ow, np.arange(w.T), act=act, alpha=alpha, limit=limit, bgu=bgu,
                                         bd=bd)
    pb.assert_close_rel_max(r["y"].float().cpu().numpy(), yref, TOL, f"forward {name}")
    pb.assert_close_rel_max(r["gx"].float().cpu().numpy(), gref, TOL, f"dgrad {name}")


def test_variant_full_size_gptoss_sampled(e4b):
    """gpt-oss-shaped layer (E=32, H=I=2880, top-4, FP4) with the clamped GLU and biases."""
    w = wl.GPTOSS.with_tokens(2048)
    prob = pb.build(w)
    bgu, bd = _biases(w, 70)
    r = _run(e4b, prob, 1, 1.702, 7.0, bgu, bd)
    oi, ow = _check_routing(prob, r)
    toks = _sample_tokens(w.T, 16, seed=7)
    yref, gref = pb.oracle_forward_dgrad(prob, oi, ow, toks, act=1, alpha=1.702, limit=7.0, bgu=bgu, bd=bd)
    pb.assert_close_rel_max(r["y"].float().cpu().numpy()[toks], yref, TOL, "forward")
    pb.assert_close_rel_max(r["gx"].float().cpu().numpy()[toks], gref, TOL, "dgrad")


@pytest.mark.parametrize("T", [1, 3, 8])
def test_variant_small_batches_take_the_grouped_kernels(e4b, T):
    w = pb.custom("v_small", E=8, H=256, I=256, k=2, T=T, seed=53)
    prob = pb.build(w)
    bgu, bd = _biases(w, 54)
    r = _run(e4b, prob, 1, 1.702, 7.0, bgu, bd, path=e4b.PATH_AUTO, want_dgrad=False)
    oi, ow = oracle.route(prob.logits.numpy(), w.k, w.renorm)
    assert np.array_equal(r["idx"].cpu().numpy(), oi)
    yref, _ = pb.oracle_forward_dgrad(prob, oi, ow, np.arange(T), want_dgrad=False, act=1, alpha=1.702, limit=7.0,
                                      bgu=bgu, bd=bd)
    pb.assert_close_rel_max(r["y"].float().cpu().numpy(), yref, TOL, "auto-path forward")
    with pytest.raises(e4b.E4BError) as ei:
        _run(e4b, prob, 1, 1.702, 7.0, bgu, bd, path=e4b.PATH_DECODE, want_dgrad=False)
    assert ei.value.status == e4b.E4B_ERR_UNSUPPORTED


def test_variant_router_gradient(e4b):
    w = pb.custom("v_router", E=8, H=256, I=192, k=2, T=200, seed=55)
    prob = pb.build(w)
    bgu, bd = _biases(w, 56)
    r = _run(e4b, prob, 1, 1.702, 0.8, bgu, bd, want_dgrad=False)
    go = pb.to_dev(prob.grad_out)
    dw, dl = e4b.e4b_moe_backward_router(r["d"], r["experts"], r["x"], r["idx"], r["wts"], go,
                                         router_logits=pb.to_dev(prob.logits))
    torch.cuda.synchronize()
    _check_status(e4b)
    idx = r["idx"].cpu().numpy()
    wgu, wd = pb.oracle_weights(prob)
    rdw, rdl = oracle.router_grad(prob.x.float().numpy(), prob.grad_out.float().numpy(), prob.logits.numpy(), idx,
                                  w.renorm, wgu, wd, act=1, alpha=1.702, limit=0.8, bgu=bgu, bd=bd)
    pb.assert_close_rel_max(dw.cpu().numpy(), rdw, TOL, "dw")
    pb.assert_close_rel_max(dl.cpu().numpy(), rdl, TOL, "dlogits")
