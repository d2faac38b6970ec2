"""The 8-bit blockwise storage modes ("experts4bit-qlora" 0.4.0, "Storage modes:
the support matrix": int8 a blockwise dynamic map, fp8 an e4m3 codebook) and the
bf16 passthrough, through the C ABI: GPU quantize and dequantize bit-exact
against the oracle; forward and input gradient (the grouped GEMMs take the 8-bit
stacks dequantized to bf16 one stack at a time) within max|diff| <= 1e-2 *
max|ref|."""
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


def _weights(E, o, i, cb, seed):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((E, o, i)) * 0.02).astype(np.float32)
    table = oracle.codebook8(cb)
    ok = np.flatnonzero(~np.isnan(table))
    w[0, 0, :64] = 0.0                                               # all-zero block
    w[0, 1, :64] = np.concatenate([[1.0], table[rng.choice(ok, 63)]]) * 0.03   # table values, absmax 0.03
    srt = np.unique(table[ok])
    w[0, 2, :64] = np.concatenate([[1.0], ((srt[:-1] + srt[1:]) * 0.5)[:63]]).astype(np.float32)   # midpoints
    return w


@pytest.mark.parametrize("cb", [wl.INT8, wl.FP8], ids=["int8", "fp8"])
@pytest.mark.parametrize("shape", [(3, 64, 2880), (2, 96, 256)])
def test_quantize8_and_dequantize8_bit_exact(e4b, cb, shape):
    w = _weights(*shape, cb, seed=sum(shape) + cb)
    oc, oa = oracle.quantize8(w, cb)
    gc, ga = e4b.e4b_quantize_nf4(torch.from_numpy(w).cuda(), codebook=cb)
    torch.cuda.synchronize()
    assert np.array_equal(gc.cpu().numpy(), oc)
    assert np.array_equal(ga.cpu().numpy(), oa)
    for dt, name in ((e4b.BF16, "bf16_bits"), (e4b.F32, "f32")):
        got = e4b.e4b_dequantize_nf4(torch.from_numpy(oc).cuda(), torch.from_numpy(oa).cuda(), shape, codebook=cb,
                                     out_dtype=dt)
        torch.cuda.synchronize()
        ref = oracle.dequantize8(oc, oa, shape, cb, name)
        g = got.view(torch.int16).cpu().numpy() if dt == e4b.BF16 else got.cpu().numpy()
        assert np.array_equal(g.view(np.uint8), ref.view(np.uint8)), name
    _check_status(e4b)


def _run(e4b, w, toks):
    prob = pb.build(w)
    t = {k: pb.to_dev(getattr(prob, k)) for k in ("pg", "ag", "pd", "ad")}
    absmax = w.codebook != wl.BF16_WEIGHTS
    experts = e4b.make_experts(t["pg"], t["pd"], t["ag"] if absmax else None, t["ad"] if absmax else None)
    d = e4b.make_desc(w.E, w.H, w.I, w.k, w.renorm, w.codebook, 64, e4b.PATH_AUTO)
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
    oi, ow = _check_routing(prob, dict(idx=idx, wts=wts, offs=None, perm=None))
    yref, gref = pb.oracle_forward_dgrad(prob, oi, ow, toks)
    pb.assert_close_rel_max(y.float().cpu().numpy()[toks], yref, TOL, "forward")
    pb.assert_close_rel_max(gx.float().cpu().numpy()[toks], gref, TOL, "dgrad")
    del t


@pytest.mark.parametrize("cb", [wl.INT8, wl.FP8, wl.BF16_WEIGHTS], ids=["int8", "fp8", "bf16"])
@pytest.mark.parametrize("E,H,I,k,T", [(6, 320, 192, 2, 300), (4, 256, 448, 2, 5)], ids=["medium", "T5"])
def test_8bit_and_bf16_forward_dgrad(e4b, cb, E, H, I, k, T):
    w = pb.custom(f"s{cb}", E=E, H=H, I=I, k=k, T=T, seed=81 + cb, codebook=cb)
    _run(e4b, w, np.arange(T))


def test_int8_olmoe_full_size_sampled(e4b):
    import dataclasses
    w = dataclasses.replace(wl.OLMOE, codebook=wl.INT8)
    _run(e4b, w, _sample_tokens(w.T, 16, seed=5))
