"""Pipelined host-buffer steps (e4b_pipe_*): every batch's y and grad_x must be
bit-identical to the stateless calls (e4b_moe_forward with g/u saved, then
e4b_moe_backward_dgrad) on device copies of the same inputs, whatever the order
in which the two buffer sets are reused; those calls are themselves held to the
oracle by the parity tests, and one batch is checked against the oracle here."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from bit_quantized_mixture_nf4_b200 import workloads as wl
from tests import _problems as pb
from tests.test_gpu_parity import TOL, _desc, _upload_experts

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def e4b():
    import bit_quantized_mixture_nf4_b200 as m
    m.lib
    return m


def _batch(w, seed, T):
    """Inputs of one batch (pinned host tensors) drawn with their own seed."""
    b = dataclasses.replace(w, seed=seed, T=T)
    x = wl.activations(b)
    return dict(x=x.pin_memory(), logits=wl.router_logits(b, x).contiguous().pin_memory(),
                go=wl.grad_output(b).pin_memory())


def _direct(e4b, d, experts, w, bt):
    """The stateless calls on device copies of one batch."""
    T = bt["x"].shape[0]
    x, lg, go = bt["x"].cuda(), bt["logits"].cuda(), bt["go"].cuda()
    saved = torch.empty(T * w.k, 2 * w.I, dtype=torch.bfloat16, device="cuda")
    y, idx, wts = e4b.e4b_moe_forward(d, experts, x, lg, saved_gu=saved)
    gx = e4b.e4b_moe_backward_dgrad(d, experts, x, idx, wts, go, saved_gu=saved)
    torch.cuda.synchronize()
    return y.cpu(), gx.cpu(), idx.cpu().numpy(), wts.cpu().numpy()


def test_pipe_matches_stateless_calls(e4b):
    w = pb.custom("pipe", E=8, H=256, I=192, k=2, T=300, seed=61)
    prob = pb.build(w)
    _, experts = _upload_experts(e4b, prob)
    d = _desc(e4b, w, e4b.PATH_GROUPED)
    # five submits over three batches (one shorter than T_max): both buffer sets
    # are reused, and a batch comes back after another one went through its set
    batches = [_batch(w, 610, 300), _batch(w, 620, 300), _batch(w, 630, 173)]
    order = [0, 1, 2, 0, 1]
    ref = [_direct(e4b, d, experts, w, bt) for bt in batches]
    pipe = e4b.e4b_pipe_create(d, experts, w.T)
    try:
        outs = []
        for i in order:
            bt = batches[i]
            T = bt["x"].shape[0]
            y = torch.empty(T, w.H, dtype=torch.bfloat16).pin_memory()
            gx = torch.empty(T, w.H, dtype=torch.bfloat16).pin_memory()
            e4b.e4b_pipe_submit(pipe, bt["x"], bt["logits"], bt["go"], y, gx)
            outs.append((i, y, gx))
        e4b.e4b_pipe_sync(pipe)
        for i, y, gx in outs:
            assert torch.equal(y, ref[i][0]), f"y of batch {i}"
            assert torch.equal(gx, ref[i][1]), f"grad_x of batch {i}"
        # argument errors are reported before anything is enqueued
        big = _batch(w, 640, w.T + 1)
        yb = torch.empty(w.T + 1, w.H, dtype=torch.bfloat16).pin_memory()
        with pytest.raises(e4b.E4BError):
            e4b.e4b_pipe_submit(pipe, big["x"], big["logits"], big["go"], yb, yb.clone().pin_memory())
        with pytest.raises(ValueError):
            e4b.e4b_pipe_submit(pipe, batches[0]["x"].clone(), batches[0]["logits"], batches[0]["go"],
                                outs[0][1], outs[0][2])
        e4b.e4b_pipe_sync(pipe)
    finally:
        e4b.e4b_pipe_destroy(pipe)
    # one batch against the oracle (routing, forward and input gradient, every token)
    bt, (y0, gx0, idx0, _) = batches[2], ref[2]
    oi, ow = oracle.route(bt["logits"].numpy(), w.k, w.renorm)
    assert np.array_equal(idx0, oi)
    sub = dataclasses.replace(prob, x=bt["x"], logits=bt["logits"], grad_out=bt["go"])
    yref, gref = pb.oracle_forward_dgrad(sub, oi, ow, np.arange(bt["x"].shape[0]))
    pb.assert_close_rel_max(y0.float().numpy(), yref, TOL, "pipe forward")
    pb.assert_close_rel_max(gx0.float().numpy(), gref, TOL, "pipe dgrad")
