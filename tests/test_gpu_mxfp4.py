"""Native MXFP4 storage for the gpt-oss experts ("experts4bit-qlora 0.31.1",
section "Scope": the gpt-oss experts ship MXFP4 weights), read as OCP
Microscaling Formats v1.0 MXFP4: 32-element blocks with E8M0 scales and E2M1
elements.  GPU quantize and dequantize bit-exact against the oracle; forward and
input gradient of the grouped path within max|diff| <= 1e-2 * max|ref|, with the
weights decoded in the GEMMs' dequantizing warps."""
import dataclasses

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


def _special_weights(E, o, i, seed):
    """N(0, 0.02) plus blocks that exercise the format's edges: all zeros, exact
    E2M1 values times a power of two, midpoints (ties), values above 6 * 2^X
    (saturation), tiny values whose scale clamps at 2^-127."""
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((E, o, i)) * 0.02).astype(np.float32)
    e2m1 = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float32)
    w[0, 0, :32] = 0.0
    w[0, 1, :32] = np.tile(np.concatenate([e2m1, -e2m1]), 2) * 2.0 ** -9
    w[0, 2, :32] = np.array([7.5, .25, .75, 1.25, 1.75, 2.5, 3.5, 5.0] * 4, np.float32) * 2.0 ** -5
    w[0, 3, :32] = 1e-39
    w[0, 4, 32:64] = -7.9 * 2.0 ** -3
    return w


@pytest.mark.parametrize("shape", [(3, 64, 2880), (2, 96, 256), (1, 8, 96)])
def test_mxfp4_quantize_and_dequantize_bit_exact(e4b, shape):
    w = _special_weights(*shape, seed=sum(shape))
    op, osc = oracle.quantize_mxfp4(w)
    gp, gs = e4b.e4b_quantize_mxfp4(torch.from_numpy(w).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(gp.cpu().numpy(), op)
    assert np.array_equal(gs.cpu().numpy(), osc)   # padding bytes included
    for dt, name in ((torch.bfloat16, "bf16_bits"), (torch.float32, "f32")):
        got = e4b.e4b_dequantize_mxfp4(torch.from_numpy(op).cuda(), torch.from_numpy(osc).cuda(), shape, dt)
        torch.cuda.synchronize()
        ref = oracle.dequantize_mxfp4(op, osc, shape, name)
        g = got.view(torch.int16).cpu().numpy().view(np.uint16) if dt == torch.bfloat16 else got.cpu().numpy()
        assert np.array_equal(g.view(np.uint8), ref.view(np.uint8)), name
    _check_status(e4b)


def _experts(e4b, prob, bgu=None, bd=None):
    t = {k: pb.to_dev(getattr(prob, k)) for k in ("pg", "ag", "pd", "ad")}
    tb = None if bgu is None else pb.to_dev(bgu)
    td = None if bd is None else pb.to_dev(bd)
    ex = e4b.make_experts(t["pg"], t["pd"], None, None, tb, td, gate_up_scales=t["ag"], down_scales=t["ad"])
    return ex, (t, tb, td)


def _run(e4b, w, toks, act=0, limit=7.0, biases=None, path=None):
    prob = pb.build(w)
    bgu, bd = biases if biases is not None else (None, None)
    experts, keep = _experts(e4b, prob, bgu, bd)
    d = e4b.make_desc(w.E, w.H, w.I, w.k, w.renorm, wl.MXFP4, 32, e4b.PATH_GROUPED if path is None else path, act,
                      1.702, limit)
    x = pb.to_dev(prob.x)
    lg = pb.to_dev(prob.logits)
    go = pb.to_dev(prob.grad_out)
    saved = torch.empty(w.T * w.k, 2 * w.I, dtype=torch.bfloat16, device="cuda")
    y, idx, wts = e4b.e4b_moe_forward(d, experts, x, lg, saved_gu=saved)
    gx = e4b.e4b_moe_backward_dgrad(d, experts, x, idx, wts, go, saved_gu=saved)
    gx_re = e4b.e4b_moe_backward_dgrad(d, experts, x, idx, wts, go)
    torch.cuda.synchronize()
    _check_status(e4b)
    assert torch.equal(gx, gx_re)
    r = dict(idx=idx, wts=wts, offs=None, perm=None)
    oi, ow = _check_routing(prob, r)
    yref, gref = pb.oracle_forward_dgrad(prob, oi, ow, toks, act=act, limit=limit, bgu=bgu, bd=bd)
    pb.assert_close_rel_max(y.float().cpu().numpy()[toks], yref, TOL, "MXFP4 forward")
    pb.assert_close_rel_max(gx.float().cpu().numpy()[toks], gref, TOL, "MXFP4 dgrad")
    return keep


@pytest.mark.parametrize("E,H,I,k,T", [(6, 320, 192, 2, 300), (4, 2880, 576, 4, 64)])
def test_mxfp4_forward_dgrad_medium(e4b, E, H, I, k, T):
    w = pb.custom("mx", E=E, H=H, I=I, k=k, T=T, seed=71 + E, codebook=wl.MXFP4)
    _run(e4b, w, np.arange(T))


def test_mxfp4_gptoss_variant_full_size_sampled(e4b):
    """The gpt-oss-shaped layer (E=32, H=I=2880, top-4) at T=2048 in native MXFP4
    with the clamped GLU and per-expert biases, sampled tokens."""
    from tests.test_gpu_variant import _biases
    w = dataclasses.replace(wl.GPTOSS, codebook=wl.MXFP4)
    _run(e4b, w, _sample_tokens(w.T, 16, seed=9), act=1, limit=7.0, biases=_biases(w, 72))


def test_mxfp4_small_batches_take_the_grouped_kernels(e4b):
    w = pb.custom("mx_small", E=8, H=256, I=256, k=2, T=3, seed=73, codebook=wl.MXFP4)
    _run(e4b, w, np.arange(3), path=e4b.PATH_AUTO)
    with pytest.raises(e4b.E4BError) as ei:
        _run(e4b, w, np.arange(3), path=e4b.PATH_DECODE)
    assert ei.value.status == e4b.E4B_ERR_UNSUPPORTED
