"""The no-allocation forward (e4b_moe_forward_noalloc) against the regular
forward (e4b_moe_forward) and the oracle.

The no-allocation entry point serves callers that cannot give the library
device memory: its scratch is a fixed array inside the library instead of a
caller workspace.  It runs the same deterministic kernels as the regular
forward, so its output must equal the regular forward's bit for bit, call after
call (the scratch is shared and reused), and match the oracle within the
forward tolerance max|diff| <= 1e-2 * max|ref|.  A second call must not change
the device's free memory.  Kept in a file of its own that is collected last."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from bit_quantized_mixture_nf4_b200 import workloads as wl
from tests import _problems as pb

pytestmark = pytest.mark.gpu

TOL = 1e-2
SCRATCH = 32 << 20   # the library's fixed scratch


@pytest.fixture(scope="module")
def e4b():
    import bit_quantized_mixture_nf4_b200 as m
    m.lib
    return m


def _layer(e4b, w, prob=None):
    """Device weights: quantized on the GPU from weights drawn there, or (prob given)
    the oracle's own packed bytes of the host-drawn weights."""
    if prob is not None:
        pg, ag, pd, ad = (pb.to_dev(getattr(prob, k)) for k in ("pg", "ag", "pd", "ad"))
    else:
        gu, dn = wl.weights(w, device=torch.device("cuda"))
        pg, ag = e4b.e4b_quantize_nf4(gu, codebook=w.codebook)
        pd, ad = e4b.e4b_quantize_nf4(dn, codebook=w.codebook)
    keep = (pg, ag, pd, ad)
    return keep, e4b.make_experts(pg, pd, ag, ad)


def _outputs(w):
    dev = torch.device("cuda")
    return (torch.empty(w.T, w.H, dtype=torch.bfloat16, device=dev),
            torch.empty(w.T, w.k, dtype=torch.int32, device=dev),
            torch.empty(w.T, w.k, dtype=torch.float32, device=dev))


def _run_pair(e4b, w, path, prob=None):
    keep, experts = _layer(e4b, w, prob)
    desc = e4b.make_desc(w.E, w.H, w.I, w.k, w.renorm, w.codebook, 64, path)
    x = wl.activations(w).cuda()
    logits = wl.router_logits(w, wl.activations(w)).cuda()
    ref, ref_idx, ref_w = e4b.e4b_moe_forward(desc, experts, x, logits)
    torch.cuda.synchronize()
    y, idx, wts = _outputs(w)
    free = []
    for _ in range(2):   # the shared scratch keeps the previous call's contents
        y.fill_(float("nan"))
        e4b.e4b_moe_forward_noalloc(desc, experts, x, logits, idx, wts, y)
        torch.cuda.synchronize()
        free.append(torch.cuda.mem_get_info()[0])
        assert torch.equal(idx, ref_idx)
        assert torch.equal(wts, ref_w)
        assert torch.equal(y, ref)
    # after the first call (which may load the library's device code), a call
    # takes no device memory
    assert free[1] == free[0]
    # routing given as input instead of logits
    y2, _, _ = e4b.e4b_moe_forward_noalloc(desc, experts, x, None, ref_idx.clone(), ref_w.clone())
    torch.cuda.synchronize()
    assert torch.equal(y2, ref)
    assert e4b.e4b_device_status() == e4b.E4B_OK
    return desc, y, idx, wts


@pytest.mark.parametrize("w,path", [(wl.TINY, 1), (wl.TINY.with_tokens(5), 0),
                                    (wl.OLMOE.with_tokens(40), 1)], ids=["tiny", "tiny-decode", "olmoe-T40"])
def test_noalloc_forward_matches_forward_two_calls(e4b, w, path):
    _run_pair(e4b, w, path)


def test_noalloc_forward_matches_oracle(e4b):
    """The tiny layer through the no-allocation entry point against the oracle
    (the oracle quantizes the same seeded weights itself)."""
    w = wl.TINY
    prob = pb.build(w)
    _, y, idx, wts = _run_pair(e4b, w, 1, prob)
    oi, ow = oracle.route(prob.logits.numpy(), w.k, w.renorm)
    assert np.array_equal(idx.cpu().numpy(), oi)
    yref, _ = pb.oracle_forward_dgrad(prob, oi, ow, np.arange(w.T), want_dgrad=False)
    pb.assert_close_rel_max(y.float().cpu().numpy(), yref, TOL, "y (no-alloc)")


def test_noalloc_near_its_scratch_limit(e4b):
    """A request whose workspace is just under the 32 MiB scratch uses the end of
    the array; it must still equal the regular forward."""
    base = wl.OLMOE
    desc = e4b.make_desc(base.E, base.H, base.I, base.k, base.renorm, base.codebook, 64, 1)
    T = 1
    while e4b.e4b_moe_workspace_size(desc, T + 1) <= SCRATCH:
        T += 1
    need = e4b.e4b_moe_workspace_size(desc, T)
    assert SCRATCH - need < SCRATCH // 16, (T, need)
    _run_pair(e4b, base.with_tokens(T), 1)


def test_noalloc_rejects_requests_larger_than_its_scratch(e4b):
    w = wl.OLMOE
    desc = e4b.make_desc(w.E, w.H, w.I, w.k, w.renorm, w.codebook, 64, 1)
    assert e4b.e4b_moe_workspace_size(desc, 4096) > SCRATCH
    ex = e4b.e4b_experts(16, 16, 16, 16)   # never dereferenced: rejected before any launch
    st = e4b.lib.e4b_moe_forward_noalloc(ctypes.byref(desc), ctypes.byref(ex), 16, 4096, None, 16, 16, 16, None)
    assert st == e4b.E4B_ERR_WORKSPACE
