"""The no-allocation forward (e4b_moe_forward_noalloc) against the regular
forward (e4b_moe_forward).

The no-allocation entry point serves callers that cannot give the library
device memory: its scratch is a fixed array inside the library instead of a
caller workspace.  Its output must match the regular forward on the same inputs,
call after call (the scratch is shared and reused), within the forward
tolerance max|diff| <= 1e-2 * max|ref|.  Kept in a file of its own that is
collected last."""
import ctypes

import numpy as np
import pytest
import torch

from bit_quantized_mixture_nf4_b200 import workloads as wl

pytestmark = pytest.mark.gpu

TOL = 1e-2


@pytest.fixture(scope="module")
def e4b():
    import bit_quantized_mixture_nf4_b200 as m
    m.lib
    return m


def _layer(e4b, w):
    dev = torch.device("cuda")
    gu, dn = wl.weights(w, device=dev)
    pg, ag = e4b.e4b_quantize_nf4(gu, codebook=w.codebook)
    pd, ad = e4b.e4b_quantize_nf4(dn, codebook=w.codebook)
    keep = (pg, ag, pd, ad)
    return keep, e4b.make_experts(pg, pd, ag, ad)


def _close(got, ref):
    got = got.float().cpu().numpy()
    ref = ref.float().cpu().numpy()
    return np.abs(got - ref).max() <= TOL * np.abs(ref).max()


@pytest.mark.parametrize("w,path", [(wl.TINY, 1), (wl.TINY.with_tokens(5), 0),
                                    (wl.OLMOE.with_tokens(40), 1)], ids=["tiny", "tiny-decode", "olmoe-T40"])
def test_noalloc_forward_matches_forward_two_calls(e4b, w, path):
    keep, experts = _layer(e4b, w)
    desc = e4b.make_desc(w.E, w.H, w.I, w.k, w.renorm, w.codebook, 64, path)
    x = wl.activations(w).cuda()
    logits = wl.router_logits(w, wl.activations(w)).cuda()
    ref, ref_idx, ref_w = e4b.e4b_moe_forward(desc, experts, x, logits)
    torch.cuda.synchronize()
    for _ in range(2):   # the shared scratch keeps the previous call's contents
        y, idx, wts = e4b.e4b_moe_forward_noalloc(desc, experts, x, logits)
        torch.cuda.synchronize()
        assert torch.equal(idx, ref_idx)
        assert torch.equal(wts, ref_w)
        assert _close(y, ref)
    # routing given as input instead of logits
    y2, _, _ = e4b.e4b_moe_forward_noalloc(desc, experts, x, None, ref_idx.clone(), ref_w.clone())
    torch.cuda.synchronize()
    assert _close(y2, ref)
    assert e4b.e4b_device_status() == e4b.E4B_OK


def test_noalloc_rejects_requests_larger_than_its_scratch(e4b):
    w = wl.OLMOE
    desc = e4b.make_desc(w.E, w.H, w.I, w.k, w.renorm, w.codebook, 64, 1)
    assert e4b.e4b_moe_workspace_size(desc, 4096) > 32 << 20
    ex = e4b.e4b_experts(16, 16, 16, 16)   # never dereferenced: rejected before any launch
    st = e4b.lib.e4b_moe_forward_noalloc(ctypes.byref(desc), ctypes.byref(ex), 16, 4096, None, 16, 16, 16, None)
    assert st == e4b.E4B_ERR_WORKSPACE
