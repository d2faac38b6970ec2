"""One fixed scenario of the expert layer for the debug-build comparison
(tests/test_gpu_debug_checks.py runs it in a child process per library build).

    python tests/_debug_run.py OUT.npz

Loads whichever build E4B_DEBUG selects, runs on cuda:0: a forward with routing
from logits and the full backward (input, routing-weight and logit gradients) of
an OLMoE-shaped layer at a ragged token count; a forward and input gradient with
routing given as input, some pairs naming experts outside [0, E) (dropped by
contract); and a decode-path forward.  It saves every output, the status after
each part and e4b_debug_checks() to OUT.npz."""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bit_quantized_mixture_nf4_b200 as e4b  # noqa: E402
from bit_quantized_mixture_nf4_b200 import workloads as wl  # noqa: E402


def layer(w, dev):
    gu, dn = wl.weights(w, device=dev)
    pg, ag = e4b.e4b_quantize_nf4(gu, codebook=w.codebook)
    pd, ad = e4b.e4b_quantize_nf4(dn, codebook=w.codebook)
    return (pg, ag, pd, ad), e4b.make_experts(pg, pd, ag, ad)


def main(out):
    dev = torch.device("cuda:0")
    res = {"debug_checks": np.array(int(e4b.e4b_debug_checks()))}
    w = wl.OLMOE.with_tokens(300)
    keep, ex = layer(w, dev)
    d = e4b.make_desc(w.E, w.H, w.I, w.k, w.renorm, w.codebook, 64, e4b.PATH_GROUPED)
    x = wl.activations(w).to(dev)
    logits = wl.router_logits(w, wl.activations(w)).to(dev)
    go = wl.grad_output(w).to(dev)
    saved_gu = torch.empty(w.P, 2 * w.I, dtype=torch.bfloat16, device=dev)
    saved_h = torch.empty(w.P, w.I, dtype=torch.bfloat16, device=dev)
    y, idx, wts = e4b.e4b_moe_forward(d, ex, x, logits, saved_gu=saved_gu, saved_h=saved_h)
    gx, gw, gl = e4b.e4b_moe_backward(d, ex, x, idx, wts, go, saved_gu=saved_gu, saved_h=saved_h,
                                      router_logits=logits)
    res["status_train"] = np.array(e4b.e4b_device_status())
    res["word_train"] = np.array(e4b.e4b_last_status_word())
    for n, t in (("y", y), ("idx", idx), ("wts", wts), ("gx", gx), ("gw", gw), ("gl", gl)):
        res[n] = (t.view(torch.int16) if t.dtype == torch.bfloat16 else t).cpu().numpy()

    # routing as input, with dropped pairs
    idx2 = idx.clone()
    idx2[::7, 0] = -1
    idx2[3::11, 1] = w.E + 3
    y2, _, _ = e4b.e4b_moe_forward(d, ex, x, None, idx2, wts.clone())
    gx2 = e4b.e4b_moe_backward_dgrad(d, ex, x, idx2, wts, go)
    res["status_given"] = np.array(e4b.e4b_device_status())
    res["word_given"] = np.array(e4b.e4b_last_status_word())
    res["y2"] = y2.view(torch.int16).cpu().numpy()
    res["gx2"] = gx2.view(torch.int16).cpu().numpy()

    # the small-batch decode path
    wd = wl.QWEN3.with_tokens(4)
    keep2, exd = layer(wd, dev)
    dd = e4b.make_desc(wd.E, wd.H, wd.I, wd.k, wd.renorm, wd.codebook, 64, e4b.PATH_DECODE)
    xd = wl.activations(wd).to(dev)
    yd, _, _ = e4b.e4b_moe_forward(dd, exd, xd, wl.router_logits(wd, wl.activations(wd)).to(dev))
    res["status_decode"] = np.array(e4b.e4b_device_status())
    res["yd"] = yd.view(torch.int16).cpu().numpy()
    torch.cuda.synchronize()
    np.savez(out, **res)


if __name__ == "__main__":
    main(sys.argv[1])
