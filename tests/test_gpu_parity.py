"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.  Bit-exact for packed bytes, absmax, bf16 dequantization,
routing indices, offsets and permutation; max|diff| <= 1e-2 * max|ref| for the
forward output and the input gradient (fp64 oracle, same dequantized weights)."""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_mixture_nf4_b200 import workloads as wl
from tests import _problems as pb

pytestmark = pytest.mark.gpu

TOL = 1e-2          # forward / dgrad: max|diff| <= TOL * max|ref|
W_RTOL = 1e-5       # routing weights: fp32 exp/sum on the GPU vs fp64 in the oracle


@pytest.fixture(scope="module")
def e4b():
    import bit_quantized_mixture_nf4_b200 as m
    m.lib   # loads the library or fails loudly
    return m


def _upload_experts(e4b, prob):
    t = {k: pb.to_dev(getattr(prob, k)) for k in ("pg", "ag", "pd", "ad")}
    return t, e4b.make_experts(t["pg"], t["pd"], t["ag"], t["ad"])


def _desc(e4b, w, path=0):
    return e4b.make_desc(w.E, w.H, w.I, w.k, w.renorm, w.codebook, 64, path)


def _check_status(e4b):
    assert e4b.e4b_device_status() == e4b.E4B_OK


# ------------------------------------------------------------- quantize / dequantize

QUANT_SHAPES = [
    ("tiny", 8, 256, 512, wl.NF4),
    ("ragged", 3, 320, 192, wl.NF4),
    ("fp4", 4, 192, 320, wl.FP4),
]


@pytest.mark.parametrize("name,E,H,I,cb", QUANT_SHAPES)
def test_quantize_dequantize_bit_exact(e4b, name, E, H, I, cb):
    w = pb.custom(name, E=E, H=H, I=I, codebook=cb, seed=E * 1000 + H)
    prob = pb.build(w)
    for stack, (pk, am) in ((prob.gu, (prob.pg, prob.ag)), (prob.dn, (prob.pd, prob.ad))):
        dev = pb.to_dev(stack)
        packed, absmax = e4b.e4b_quantize_nf4(dev, codebook=cb)
        assert np.array_equal(packed.cpu().numpy(), pk)
        assert np.array_equal(absmax.cpu().numpy().view(np.uint32), am.view(np.uint32))
        # dequantize the ORACLE's bytes on the GPU
        bf = e4b.e4b_dequantize_nf4(pb.to_dev(pk), pb.to_dev(am), stack.shape, codebook=cb, out_dtype=e4b.BF16)
        ref_bits = oracle.dequantize(pk, am, stack.shape, cb, "bf16_bits")
        assert np.array_equal(wl.bf16_bits(bf), ref_bits)
        f32 = e4b.e4b_dequantize_nf4(pb.to_dev(pk), pb.to_dev(am), stack.shape, codebook=cb, out_dtype=e4b.F32)
        ref32 = oracle.dequantize(pk, am, stack.shape, cb, "f32")
        assert np.array_equal(f32.cpu().numpy().view(np.uint32), ref32.view(np.uint32))
    _check_status(e4b)


@pytest.mark.parametrize("cb", [wl.NF4, wl.FP4])
def test_quantize_edge_blocks(e4b, cb):
    """Zero blocks, exact codebook values, exact midpoints (ties), -0, huge and tiny scales."""
    c = oracle.codebook(cb)
    vals = np.unique(c[[q for q in range(16) if not (cb == wl.FP4 and q == 8)]])
    mids = ((vals[:-1] + vals[1:]) * np.float32(0.5)).astype(np.float32)
    rows = np.zeros((6, 64), np.float32)
    rows[1, :16] = c                      # codebook values themselves (absmax 1)
    rows[2, 0] = 1.0
    rows[2, 1:1 + len(mids)] = mids       # ties
    rows[3, :] = -0.0
    rows[3, 5] = 3e38
    rows[3, 6] = -1e-30
    rng = np.random.default_rng(3)
    rows[4] = rng.standard_normal(64).astype(np.float32) * 1e-38
    rows[5] = rng.standard_normal(64).astype(np.float32) * 1e30
    w = rows.reshape(1, 6, 64)
    pk, am = oracle.quantize(w, cb)
    packed, absmax = e4b.e4b_quantize_nf4(pb.to_dev(w), codebook=cb)
    assert np.array_equal(packed.cpu().numpy(), pk)
    assert np.array_equal(absmax.cpu().numpy().view(np.uint32), am.view(np.uint32))
    bf = e4b.e4b_dequantize_nf4(pb.to_dev(pk), pb.to_dev(am), w.shape, codebook=cb)
    assert np.array_equal(wl.bf16_bits(bf), oracle.dequantize(pk, am, w.shape, cb, "bf16_bits"))


@pytest.mark.parametrize("shape", [(1, 1, 64), (3, 7, 128), (2, 33, 192), (5, 41, 320)])
@pytest.mark.parametrize("cb", [wl.NF4, wl.FP4])
def test_quantize_dequantize_ragged_counts(e4b, shape, cb):
    """Block and 32-element chunk counts that are not multiples of a warp's share
    (8 blocks / 32 chunks): the partial last warp stores only its own bytes."""
    rng = np.random.default_rng(shape[1])
    w = (rng.standard_normal(shape) * 0.02).astype(np.float32)
    pk, am = oracle.quantize(w, cb)
    dev = pb.to_dev(w)
    packed = torch.full((shape[0], shape[1] * shape[2] // 2 + 64), 0xAB, dtype=torch.uint8, device="cuda")
    absmax = torch.full((shape[0], shape[1] * shape[2] // 64), -1.0, dtype=torch.float32, device="cuda")
    e4b.e4b_quantize_nf4(dev, codebook=cb, packed=packed, absmax=absmax)
    got = packed.cpu().numpy().reshape(-1)
    n = pk.size
    assert np.array_equal(got[:n], pk.reshape(-1))
    assert (got[n:] == 0xAB).all()          # nothing written past the end
    assert np.array_equal(absmax.cpu().numpy().view(np.uint32), am.view(np.uint32))
    out = torch.full((w.size + 256,), 7.0, dtype=torch.bfloat16, device="cuda")
    e4b.e4b_dequantize_nf4(pb.to_dev(pk), pb.to_dev(am), shape, codebook=cb, out=out)
    bits = wl.bf16_bits(out)
    assert np.array_equal(bits[:w.size].reshape(shape), oracle.dequantize(pk, am, shape, cb, "bf16_bits"))
    assert (bits[w.size:] == wl.bf16_bits(torch.tensor([7.0], dtype=torch.bfloat16))[0]).all()
    _check_status(e4b)


@pytest.mark.parametrize("wname", ["olmoe", "qwen3", "mixtral", "gptoss"])
def test_quantize_full_size_bit_exact(e4b, wname):
    """Full-size stacks of every layer family: GPU quantize == oracle quantize on
    every block, and GPU bf16 dequantize of the oracle bytes == oracle on every element."""
    w = wl.ALL[wname]
    prob = pb.build(w)
    for stack, pk, am in ((prob.gu, prob.pg, prob.ag), (prob.dn, prob.pd, prob.ad)):
        dev = pb.to_dev(stack)
        packed, absmax = e4b.e4b_quantize_nf4(dev, codebook=w.codebook)
        del dev
        assert np.array_equal(packed.cpu().numpy(), pk)
        assert np.array_equal(absmax.cpu().numpy().view(np.uint32), am.view(np.uint32))
        bf = e4b.e4b_dequantize_nf4(pb.to_dev(pk), pb.to_dev(am), stack.shape, codebook=w.codebook)
        # sampled rows of the oracle dequantization (every element of those rows)
        rng = np.random.default_rng(1)
        E, O, In = stack.shape
        for e in rng.choice(E, size=min(E, 3), replace=False):
            rows = rng.choice(O, size=16, replace=False)
            sub_pk = pk[e].reshape(O, In // 2)[rows]
            sub_am = am[e].reshape(O, In // 64)[rows]
            ref = oracle.dequantize(sub_pk.reshape(1, -1), sub_am.reshape(1, -1), (1, 16, In), w.codebook, "bf16_bits")
            got = wl.bf16_bits(bf[e][torch.from_numpy(rows).cuda()])
            assert np.array_equal(got.reshape(1, 16, In), ref)
        del bf
    torch.cuda.empty_cache()
    _check_status(e4b)


# -------------------------------------------------------------- routing + grouping

def _run_forward(e4b, prob, path=0, route=True, save=True):
    w = prob.w
    t, experts = _upload_experts(e4b, prob)
    d = _desc(e4b, w, path)
    x = pb.to_dev(prob.x)
    T = w.T
    logits = pb.to_dev(prob.logits) if route else None
    if route:
        idx = torch.empty(T, w.k, dtype=torch.int32, device="cuda")
        wts = torch.empty(T, w.k, dtype=torch.float32, device="cuda")
    else:
        oi, ow = oracle.route(prob.logits.numpy(), w.k, w.renorm)
        idx, wts = pb.to_dev(oi), pb.to_dev(ow.astype(np.float32))
    gu = torch.empty(T * w.k, 2 * w.I, dtype=torch.bfloat16, device="cuda") if save else None
    offs = torch.empty(w.E + 1, dtype=torch.int32, device="cuda") if save else None
    perm = torch.empty(T * w.k, dtype=torch.int32, device="cuda") if save else None
    y, idx, wts = e4b.e4b_moe_forward(d, experts, x, logits, idx, wts, saved_gu=gu, offsets_out=offs, perm_out=perm)
    torch.cuda.synchronize()
    _check_status(e4b)
    return dict(t=t, experts=experts, d=d, x=x, y=y, idx=idx, wts=wts, gu=gu, offs=offs, perm=perm)


def _check_routing(prob, r):
    w = prob.w
    oi, ow = oracle.route(prob.logits.numpy(), w.k, w.renorm)
    gi = r["idx"].cpu().numpy()
    assert np.array_equal(gi, oi)
    np.testing.assert_allclose(r["wts"].cpu().numpy(), ow, rtol=W_RTOL, atol=0)
    if r["offs"] is not None:
        counts, offsets, perm = oracle.permute(oi, w.E)
        assert np.array_equal(r["offs"].cpu().numpy(), offsets)
        assert np.array_equal(r["perm"].cpu().numpy(), perm)
    return oi, ow


def _sample_tokens(T, n, seed=0):
    rng = np.random.default_rng(seed)
    if T <= n:
        return np.arange(T)
    s = rng.choice(T, size=n, replace=False)
    return np.unique(np.concatenate([s, [0, T - 1]]))


MEDIUM = [
    pb.custom("ragged", E=4, H=320, I=192, k=2, T=500, seed=11),                    # M, N and K tails
    pb.custom("skew", E=16, H=256, I=256, k=4, T=777, seed=12, router="zipf"),      # empty experts, skew
    pb.custom("fp4med", E=6, H=192, I=320, k=3, T=333, seed=13, codebook=wl.FP4),
    pb.custom("even6", E=8, H=384, I=128, k=2, T=300, seed=14),                     # 6 / 2 blocks per row
    wl.TINY,
]


@pytest.mark.parametrize("w", MEDIUM, ids=lambda w: w.name)
def test_forward_and_dgrad_medium(e4b, w):
    prob = pb.build(w)
    r = _run_forward(e4b, prob, path=e4b.PATH_GROUPED)
    oi, ow = _check_routing(prob, r)
    toks = np.arange(w.T)
    yref, gref = pb.oracle_forward_dgrad(prob, oi, ow, toks)
    pb.assert_close_rel_max(r["y"].float().cpu().numpy(), yref, TOL, "forward")
    go = pb.to_dev(prob.grad_out)
    gx = e4b.e4b_moe_backward_dgrad(r["d"], r["experts"], r["x"], r["idx"], r["wts"], go, saved_gu=r["gu"])
    torch.cuda.synchronize()
    pb.assert_close_rel_max(gx.float().cpu().numpy(), gref, TOL, "dgrad (saved g,u)")
    gx2 = e4b.e4b_moe_backward_dgrad(r["d"], r["experts"], r["x"], r["idx"], r["wts"], go, saved_gu=None)
    torch.cuda.synchronize()
    pb.assert_close_rel_max(gx2.float().cpu().numpy(), gref, TOL, "dgrad (recomputed g,u)")
    _check_status(e4b)


def _tile_edge_tokens(idx, E, k, tile_rows=256):
    """Tokens owning the first and the last grouped row of every expert's first and
    last m-tile (from the oracle's permutation): each expert's first and last tile
    then has checked rows."""
    counts, offsets, perm = oracle.permute(idx, E)
    toks = set()
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi == lo:
            continue
        last0 = lo + (hi - 1 - lo) // tile_rows * tile_rows   # first row of the last m-tile
        for row in (lo, min(lo + tile_rows, hi) - 1, last0, hi - 1):
            toks.add(int(perm[row]) // k)
    return np.array(sorted(toks), np.int64)


@pytest.mark.parametrize("wname,T", [("olmoe", 4096), ("qwen3", 8192), ("mixtral", 16384), ("gptoss", 2048)])
def test_forward_and_dgrad_full_size_sampled(e4b, wname, T):
    """Full-size layer in the launch configuration the benchmark uses; routing,
    offsets and permutation checked on every token, y and grad_x on sampled tokens:
    random ones plus the owners of the first and last rows of every expert's first
    and last m-tile."""
    w = wl.ALL[wname].with_tokens(T)
    prob = pb.build(w)
    r = _run_forward(e4b, prob, path=e4b.PATH_GROUPED)
    oi, ow = _check_routing(prob, r)
    go = pb.to_dev(prob.grad_out)
    gx = e4b.e4b_moe_backward_dgrad(r["d"], r["experts"], r["x"], r["idx"], r["wts"], go, saved_gu=r["gu"])
    torch.cuda.synchronize()
    _check_status(e4b)
    toks = np.union1d(_sample_tokens(T, 12 if wname == "mixtral" else 24, seed=T), _tile_edge_tokens(oi, w.E, w.k))
    yref, gref = pb.oracle_forward_dgrad(prob, oi, ow, toks)
    pb.assert_close_rel_max(r["y"].float().cpu().numpy()[toks], yref, TOL, "forward")
    pb.assert_close_rel_max(gx.float().cpu().numpy()[toks], gref, TOL, "dgrad")
    del r, gx
    torch.cuda.empty_cache()


@pytest.mark.parametrize("wname,T", [("qwen3", 1), ("qwen3", 2), ("qwen3", 4), ("qwen3", 8), ("gptoss", 1),
                                     ("tiny", 3)])
def test_decode_path(e4b, wname, T):
    """T <= 8: the weight-streaming decode kernels vs the oracle, and vs the grouped path."""
    w = wl.ALL[wname].with_tokens(T)
    prob = pb.build(w)
    r = _run_forward(e4b, prob, path=e4b.PATH_DECODE, save=False)
    oi, ow = _check_routing(prob, r)
    yref, _ = pb.oracle_forward_dgrad(prob, oi, ow, np.arange(T), want_dgrad=False)
    pb.assert_close_rel_max(r["y"].float().cpu().numpy(), yref, TOL, "decode forward")
    rg = _run_forward(e4b, prob, path=e4b.PATH_GROUPED, save=False)
    pb.assert_close_rel_max(rg["y"].float().cpu().numpy(), yref, TOL, "grouped forward")


@pytest.mark.parametrize("E,H,I,k,T,cb", [(4, 512, 256, 1, 1, wl.NF4), (4, 512, 256, 1, 3, wl.FP4),
                                            (6, 192, 320, 2, 5, wl.NF4), (16, 4096, 128, 2, 1, wl.NF4)])
def test_decode_small_shapes(e4b, E, H, I, k, T, cb):
    """Decode path where fewer than 8 (slot, tile) units exist per CTA (K split over
    warps), K not a multiple of the per-warp split, and 16 output rows per CTA."""
    w = pb.custom("dec", E=E, H=H, I=I, k=k, T=T, seed=31 + T, codebook=cb)
    prob = pb.build(w)
    r = _run_forward(e4b, prob, path=e4b.PATH_DECODE, save=False)
    oi, ow = _check_routing(prob, r)
    yref, _ = pb.oracle_forward_dgrad(prob, oi, ow, np.arange(T), want_dgrad=False)
    pb.assert_close_rel_max(r["y"].float().cpu().numpy(), yref, TOL, "decode forward")


def test_decode_given_routing_repeats_and_invalid(e4b):
    """Caller-given routing on the decode path: an expert chosen twice by one token,
    one expert taking more than 8 pairs (two slots), and an out-of-range id (that
    pair contributes nothing).  Same result from the grouped path."""
    w = pb.custom("dec-given", E=8, H=256, I=128, k=2, T=8, seed=41)
    prob = pb.build(w)
    idx = np.zeros((8, 2), np.int32)
    idx[3] = (-1, 5)
    idx[5] = (7, 0)
    rng = np.random.default_rng(5)
    wts = rng.uniform(0.1, 1.0, size=(8, 2)).astype(np.float32)
    ref_idx = idx.copy()
    ref_w = wts.astype(np.float64)
    ref_idx[3, 0] = 0          # the out-of-range pair: weight 0 on a valid expert adds nothing
    ref_w[3, 0] = 0.0
    yref, _ = pb.oracle_forward_dgrad(prob, ref_idx, ref_w, np.arange(8), want_dgrad=False)
    t, experts = _upload_experts(e4b, prob)
    x = pb.to_dev(prob.x)
    for path in (e4b.PATH_DECODE, e4b.PATH_GROUPED):
        d = _desc(e4b, w, path)
        y, gi, gw = e4b.e4b_moe_forward(d, experts, x, None, pb.to_dev(idx), pb.to_dev(wts))
        torch.cuda.synchronize()
        _check_status(e4b)
        assert np.array_equal(gi.cpu().numpy(), idx)   # given routing is left as it was
        pb.assert_close_rel_max(y.float().cpu().numpy(), yref, TOL, f"forward path {path}")


def test_given_routing_and_zero_tokens(e4b):
    w = pb.custom("given", E=8, H=256, I=128, k=2, T=200, seed=21)
    prob = pb.build(w)
    r = _run_forward(e4b, prob, path=e4b.PATH_GROUPED, route=False)
    oi, ow = oracle.route(prob.logits.numpy(), w.k, w.renorm)
    yref, _ = pb.oracle_forward_dgrad(prob, oi, ow.astype(np.float32).astype(np.float64), np.arange(w.T), False)
    pb.assert_close_rel_max(r["y"].float().cpu().numpy(), yref, TOL, "forward with given routing")
    # T == 0 is a no-op
    empty = torch.empty(0, w.H, dtype=torch.bfloat16, device="cuda")
    y0, _, _ = e4b.e4b_moe_forward(r["d"], r["experts"], empty, None,
                                   torch.empty(0, w.k, dtype=torch.int32, device="cuda"),
                                   torch.empty(0, w.k, dtype=torch.float32, device="cuda"))
    assert y0.shape == (0, w.H)


def test_single_expert_dense_mlp(e4b):
    """E=1, k=1: the layer is a dense SwiGLU MLP with weight 1 (softmax over one expert)."""
    w = pb.custom("dense", E=1, H=256, I=256, k=1, T=130, seed=22)
    prob = pb.build(w)
    r = _run_forward(e4b, prob, path=e4b.PATH_GROUPED)
    assert np.all(r["wts"].cpu().numpy() == 1.0)
    oi, ow = _check_routing(prob, r)
    yref, gref = pb.oracle_forward_dgrad(prob, oi, ow, np.arange(w.T))
    pb.assert_close_rel_max(r["y"].float().cpu().numpy(), yref, TOL, "dense forward")


def test_consecutive_shapes_share_workspace(e4b):
    """Back-to-back grouped forwards of different layers through one workspace:
    the second call's routing, grouping and output must not see anything the
    first call left in the workspace (or in any cache in front of it)."""
    ws_shapes = [pb.custom("seqA", E=16, H=256, I=192, k=4, T=700, seed=41),
                 pb.custom("seqB", E=6, H=320, I=128, k=2, renorm=False, T=450, seed=42),
                 pb.custom("seqC", E=16, H=256, I=192, k=3, T=523, seed=43)]
    probs = [pb.build(w) for w in ws_shapes]
    size = max(e4b.e4b_moe_workspace_size(_desc(e4b, w, e4b.PATH_GROUPED), w.T) for w in ws_shapes)
    ws = torch.empty(size, dtype=torch.uint8, device="cuda")
    for rnd in range(2):
        for w, prob in zip(ws_shapes, probs):
            _, experts = _upload_experts(e4b, prob)
            d = _desc(e4b, w, e4b.PATH_GROUPED)
            x, logits = pb.to_dev(prob.x), pb.to_dev(prob.logits)
            offs = torch.empty(w.E + 1, dtype=torch.int32, device="cuda")
            perm = torch.empty(w.T * w.k, dtype=torch.int32, device="cuda")
            y, idx, wts = e4b.e4b_moe_forward(d, experts, x, logits, offsets_out=offs, perm_out=perm, ws=ws)
            torch.cuda.synchronize()
            _check_status(e4b)
            oi, ow = _check_routing(prob, dict(idx=idx, wts=wts, offs=offs, perm=perm))
            yref, _ = pb.oracle_forward_dgrad(prob, oi, ow, np.arange(w.T), want_dgrad=False)
            pb.assert_close_rel_max(y.float().cpu().numpy(), yref, TOL, f"forward {w.name} (pass {rnd})")
