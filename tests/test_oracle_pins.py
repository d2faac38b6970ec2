"""Pins for the CPU oracle: each test checks the oracle against something other
than itself -- a published construction, a closed form, an invariant the pages
state, a library routine, brute force, or finite differences.  CPU only."""
import os

import numpy as np
import pytest
import torch

import oracle
from bit_quantized_mixture_nf4_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "fidelity_bounds.txt")


def golden():
    out = {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, v = line.split()[:2]
        out[k] = float(v)
    return out


# ---------------------------------------------------------------- codebooks

def test_nf4_codebook_matches_normalfloat_construction():
    """NF4 = quantiles of N(0,1) (QLoRA's NormalFloat): 8 positive values from
    ppf(linspace(d, 1/2, 9)[:-1]), 7 negative from -ppf(linspace(d, 1/2, 8)[:-1]),
    zero, normalised by the maximum; d = (1 - 1/30 + 1 - 1/32) / 2."""
    from scipy.stats import norm
    d = 0.5 * ((1 - 1 / 30) + (1 - 1 / 32))
    pos = norm.ppf(np.linspace(d, 0.5, 9)[:-1])
    neg = -norm.ppf(np.linspace(d, 0.5, 8)[:-1])
    v = np.sort(np.concatenate([pos, [0.0], neg]))
    v = v / v.max()
    c = oracle.codebook(oracle.NF4).astype(np.float64)
    assert np.all(np.diff(c) > 0)
    assert c[0] == -1.0 and c[7] == 0.0 and c[15] == 1.0
    np.testing.assert_allclose(c, v, atol=5e-7, rtol=0)


def test_fp4_codebook_is_e2m1_over_six():
    c = oracle.codebook(oracle.FP4).astype(np.float64)
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6]) / 6.0
    np.testing.assert_allclose(c[:8], mags, rtol=1e-7)
    np.testing.assert_allclose(c[8:], -mags, rtol=1e-7)
    assert np.signbit(c[8])   # code 0b1000 is -0 (never produced by quantize)


# ----------------------------------------------------------- bf16 rounding

def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    v = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 20000),
        # exact ties: low half exactly 0x8000 with even and odd upper halves
        (np.arange(2000, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
        np.array([0.0, -0.0, np.inf, -np.inf, 3.4e38, 1e-45, -1e-45], np.float32),
    ]).astype(np.float32)
    v = v[np.isfinite(v) | np.isinf(v)]
    ours = oracle.f32_to_bf16_bits(v)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


# ------------------------------------------------------ quantize / dequantize

def _blocks(n_blocks, scale=0.02, seed=0):
    rng = np.random.default_rng(seed)
    s = scale * np.exp(rng.uniform(-3, 3, (n_blocks, 1)))
    return (rng.standard_normal((n_blocks, 64)) * s).astype(np.float32)


@pytest.mark.parametrize("cb,half_gap", [(oracle.NF4, (1.0 - 0.6961928009986877) / 2), (oracle.FP4, 1.0 / 6.0)])
def test_roundtrip_error_bound(cb, half_gap):
    """|w - deq| <= absmax * (largest codebook gap)/2 per element (plus fp32 rounding)."""
    w = _blocks(4096, seed=1).reshape(8, 512, 64)
    packed, absmax = oracle.quantize(w, cb)
    deq = oracle.dequantize(packed, absmax, w.shape, cb, "f32")
    a = absmax.reshape(8, 512, 1)
    err = np.abs(w.astype(np.float64) - deq.astype(np.float64))
    bound = a * half_gap * (1 + 1e-6) + np.abs(w) * 2.0 ** -23
    assert np.all(err <= bound)
    # bf16 output adds at most half a bf16 ulp of the value
    deq16 = oracle.dequantize(packed, absmax, w.shape, cb, "bf16")
    assert np.all(np.abs(deq16 - deq) <= np.abs(deq) * 2.0 ** -8)


@pytest.mark.parametrize("cb", [oracle.NF4, oracle.FP4])
def test_exact_reproduction_of_codebook_values_and_zeros(cb):
    c = oracle.codebook(cb)
    codes = list(range(16)) if cb == oracle.NF4 else [q for q in range(16) if q != 8]
    rng = np.random.default_rng(2)
    for a in (1.0, 0.02, 3.7e-3, 117.0):
        a = np.float32(a)
        vals = np.array([np.float32(c[q]) * a for q in codes], np.float32)
        block = np.zeros(64, np.float32)
        pos = rng.permutation(64)[: len(vals)]
        block[pos] = vals
        packed, absmax = oracle.quantize(block.reshape(1, 1, 64), cb)
        assert absmax[0, 0] == a
        deq = oracle.dequantize(packed, absmax, (1, 1, 64), cb, "f32").ravel()
        assert np.array_equal(deq[pos], vals)
        zero_code = 7 if cb == oracle.NF4 else 0
        nib = np.stack([packed[0] >> 4, packed[0] & 15], 1).ravel()
        assert np.array_equal(nib[pos], np.array(codes))
        rest = np.setdiff1d(np.arange(64), pos)
        assert np.all(nib[rest] == zero_code)
        assert np.all(deq[rest] == 0) and not np.any(np.signbit(deq[rest]))


@pytest.mark.parametrize("cb", [oracle.NF4, oracle.FP4])
def test_all_zero_block(cb):
    packed, absmax = oracle.quantize(np.zeros((2, 3, 64), np.float32), cb)
    zero_byte = 0x77 if cb == oracle.NF4 else 0x00
    assert np.all(packed == zero_byte) and np.all(absmax == 0)
    assert np.all(oracle.dequantize(packed, absmax, (2, 3, 64), cb, "f32") == 0)


def test_nibble_order_first_element_high():
    """The first element of each pair goes to the high nibble."""
    block = np.zeros((1, 1, 64), np.float32)
    block[0, 0, 0] = 1.0      # +absmax -> NF4 code 15
    block[0, 0, 3] = -1.0     # -absmax -> NF4 code 0
    packed, absmax = oracle.quantize(block, oracle.NF4)
    assert packed[0, 0] == 0xF7 and packed[0, 1] == 0x70


@pytest.mark.parametrize("cb", [oracle.NF4, oracle.FP4])
def test_idempotent(cb):
    w = _blocks(2048, seed=3).reshape(4, 256, 128)
    packed, absmax = oracle.quantize(w, cb)
    deq = oracle.dequantize(packed, absmax, w.shape, cb, "f32")
    p2, a2 = oracle.quantize(deq, cb)
    assert np.array_equal(a2, absmax)
    assert np.array_equal(p2, packed)


@pytest.mark.parametrize("cb", [oracle.NF4, oracle.FP4])
def test_tie_goes_to_smaller_value(cb):
    c = oracle.codebook(cb)
    vals = np.unique(c[[q for q in range(16) if not (cb == oracle.FP4 and q == 8)]])
    mids = ((vals[:-1] + vals[1:]) * np.float32(0.5)).astype(np.float32)
    block = np.zeros(64, np.float32)
    block[0] = 1.0
    block[1:1 + len(mids)] = mids
    packed, absmax = oracle.quantize(block.reshape(1, 1, 64), cb)
    deq = oracle.dequantize(packed, absmax, (1, 1, 64), cb, "f32").ravel()
    assert np.array_equal(deq[1:1 + len(mids)], vals[:-1])


def test_blocksize_validation():
    """in_features must be a multiple of the block size (64)."""
    with pytest.raises(oracle.OracleError) as ei:
        oracle.quantize(np.zeros((1, 2, 96), np.float32))
    assert ei.value.code == 2
    with pytest.raises(oracle.OracleError):
        oracle.quantize(np.zeros((1, 2, 64), np.float32), blocksize=32)


def test_error_ordering_nf4_below_fp4():
    """NF4 reconstructs ~Gaussian weights better than FP4."""
    rng = np.random.default_rng(4)
    w = (rng.standard_normal((4, 1024, 64)) * 0.02).astype(np.float32)
    errs = {}
    for cb in (oracle.NF4, oracle.FP4):
        p, a = oracle.quantize(w, cb)
        d = oracle.dequantize(p, a, w.shape, cb, "f32")
        errs[cb] = np.sqrt(np.mean((d - w) ** 2) / np.mean(w ** 2))
    assert errs[oracle.NF4] < errs[oracle.FP4]


def test_nf4_dequant_mean_abs_error_bound():
    g = golden()
    rng = np.random.default_rng(5)
    w = (rng.standard_normal((2, 512, 256)) * 0.02).astype(np.float32)
    p, a = oracle.quantize(w)
    d = oracle.dequantize(p, a, w.shape, oracle.NF4, "bf16")
    assert np.mean(np.abs(d - w)) <= g["nf4_dequant_mean_abs_bound"]


# -------------------------------------------------------------- routing

def _logits(T, E, seed):
    rng = np.random.default_rng(seed)
    l = rng.standard_normal((T, E)).astype(np.float32)
    l[::7, 3] = l[::7, 5]           # exact ties between experts 3 and 5
    return l


@pytest.mark.parametrize("E,k,renorm", [(8, 2, True), (64, 8, False), (128, 8, True), (32, 4, True)])
def test_route_brute_force(E, k, renorm):
    T = 97
    l = _logits(T, E, E + k)
    idx, w = oracle.route(l, k, renorm)
    for t in range(T):
        order = np.lexsort((np.arange(E), -l[t].astype(np.float64)))   # logit desc, index asc
        assert np.array_equal(idx[t], order[:k])
        ld = l[t].astype(np.float64)
        z = np.exp(ld - ld.max()).sum()
        sel = ld[idx[t]]
        # softmax ratios are exp of logit differences
        np.testing.assert_allclose(w[t] / w[t][0], np.exp(sel - sel[0]), rtol=1e-12)
        if renorm:
            assert abs(w[t].sum() - 1.0) < 1e-12
        else:
            np.testing.assert_allclose(w[t][0], 1.0 / z, rtol=1e-12)


def test_permute_invariants():
    T, E, k = 300, 16, 4
    l = _logits(T, E, 7)
    idx, _ = oracle.route(l, k, True)
    counts, offsets, perm = oracle.permute(idx, E)
    flat = idx.ravel()
    assert np.array_equal(counts, np.bincount(flat, minlength=E))
    assert offsets[0] == 0 and offsets[-1] == T * k and np.all(np.diff(offsets) >= 0)
    assert np.array_equal(np.sort(perm), np.arange(T * k))
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert np.all(flat[seg] == e)
        assert np.all(np.diff(seg) > 0)          # ascending pair id == ascending token


# -------------------------------------------------------------- forward

def _tiny_problem(E=4, H=64, I=64, T=8, k=2, seed=9, renorm=True):
    rng = np.random.default_rng(seed)
    x = torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)).to(torch.bfloat16).float().numpy()
    gu = (rng.standard_normal((E, 2 * I, H)) * 0.05).astype(np.float32)
    dn = (rng.standard_normal((E, H, I)) * 0.05).astype(np.float32)
    pg, ag = oracle.quantize(gu)
    pd, ad = oracle.quantize(dn)
    wgu = oracle.dequantize(pg, ag, gu.shape)
    wd = oracle.dequantize(pd, ad, dn.shape)
    l = rng.standard_normal((T, E)).astype(np.float32)
    idx, w = oracle.route(l, k, renorm)
    return x, idx, w, wgu, wd, gu, dn


def _dense_reference(x, idx, w, wgu, wd):
    """Every expert on every token in fp64 (einsum), then masked by routing."""
    E, I2, H = wgu.shape
    I = I2 // 2
    xd = x.astype(np.float64)
    G = np.einsum("th,eih->eti", xd, wgu[:, :I].astype(np.float64))
    U = np.einsum("th,eih->eti", xd, wgu[:, I:].astype(np.float64))
    Hh = G / (1 + np.exp(-G)) * U
    Y = np.einsum("eti,ehi->eth", Hh, wd.astype(np.float64))
    T = x.shape[0]
    gate = np.zeros((E, T))
    for t in range(T):
        for j in range(idx.shape[1]):
            gate[idx[t, j], t] += w[t, j]
    return np.einsum("et,eth->th", gate, Y)


def test_forward_matches_dense_fp64_reference():
    x, idx, w, wgu, wd, *_ = _tiny_problem(E=6, H=128, I=64, T=24, k=3)
    y = oracle.forward(x, idx, w, wgu, wd)
    ref = _dense_reference(x, idx, w, wgu, wd)
    np.testing.assert_allclose(y, ref, rtol=1e-10, atol=1e-12 * np.abs(ref).max())
    # same-weights tolerance on the pages is 1e-4; fp64 is far inside it
    assert np.abs(y - ref).max() <= golden()["forward_same_weights_tolerance"] * np.abs(ref).max()
    sub = np.array([5, 0, 17])
    np.testing.assert_array_equal(oracle.forward(x, idx, w, wgu, wd, tokens=sub), y[sub])


def test_forward_single_expert_is_dense_swiglu_mlp():
    x, _, _, wgu, wd, *_ = _tiny_problem(E=1, H=64, I=128, T=5, k=1)
    idx = np.zeros((5, 1), np.int32)
    w = np.ones((5, 1))
    y = oracle.forward(x, idx, w, wgu, wd)
    xt = torch.from_numpy(x).double()
    g = xt @ torch.from_numpy(wgu[0, :128]).double().t()
    u = xt @ torch.from_numpy(wgu[0, 128:]).double().t()
    ref = (torch.nn.functional.silu(g) * u) @ torch.from_numpy(wd[0]).double().t()
    np.testing.assert_allclose(y, ref.numpy(), rtol=1e-10, atol=1e-13)


@pytest.mark.parametrize("cb,key", [(oracle.NF4, "nf4_forward_relerr_cap"), (oracle.FP4, "fp4_forward_relerr_cap")])
def test_forward_relerr_vs_true_weights_within_page_caps(cb, key):
    """Forward with quantized weights vs the true fp32 weights stays under the
    per-scheme ceilings the pages print, and NF4 < FP4."""
    g = golden()
    rng = np.random.default_rng(11)
    E, H, I, T, k = 8, 256, 512, 64, 2
    x = torch.from_numpy(rng.standard_normal((T, H)).astype(np.float32)).to(torch.bfloat16).float().numpy()
    gu = (rng.standard_normal((E, 2 * I, H)) * 0.02).astype(np.float32)
    dn = (rng.standard_normal((E, H, I)) * 0.02).astype(np.float32)
    idx, w = oracle.route(rng.standard_normal((T, E)).astype(np.float32), k, True)
    ref = oracle.forward(x, idx, w, gu, dn)
    errs = {}
    for c in (oracle.NF4, oracle.FP4):
        pg, ag = oracle.quantize(gu, c)
        pd, ad = oracle.quantize(dn, c)
        y = oracle.forward(x, idx, w, oracle.dequantize(pg, ag, gu.shape, c), oracle.dequantize(pd, ad, dn.shape, c))
        errs[c] = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert errs[cb] <= g[key]
    assert errs[oracle.NF4] <= g["nf4_forward_relerr_true_weights_bound"]
    assert errs[oracle.NF4] < errs[oracle.FP4]


# -------------------------------------------------------------- dgrad

def test_dgrad_matches_central_finite_differences():
    x, idx, w, wgu, wd, *_ = _tiny_problem(E=4, H=64, I=64, T=8, k=2)
    rng = np.random.default_rng(12)
    go = rng.standard_normal(x.shape)
    gx = oracle.dgrad(x, go, idx, w, wgu, wd)
    eps = 1e-6
    num = np.zeros_like(gx)
    for t in range(x.shape[0]):
        for c in range(x.shape[1]):
            xp = x.astype(np.float64).copy()
            xm = xp.copy()
            xp[t, c] += eps
            xm[t, c] -= eps
            fp = (oracle.forward(xp, idx, w, wgu, wd, tokens=[t]) * go[t]).sum()
            fm = (oracle.forward(xm, idx, w, wgu, wd, tokens=[t]) * go[t]).sum()
            num[t, c] = (fp - fm) / (2 * eps)
    np.testing.assert_allclose(gx, num, rtol=1e-6, atol=1e-6 * np.abs(num).max())


def test_dgrad_adjoint_identity():
    """<grad_out, J v> = <dgrad(grad_out), v> with J v by a central difference."""
    x, idx, w, wgu, wd, *_ = _tiny_problem(E=5, H=128, I=64, T=16, k=3, seed=13)
    rng = np.random.default_rng(14)
    go = rng.standard_normal(x.shape)
    v = rng.standard_normal(x.shape)
    eps = 1e-5
    xd = x.astype(np.float64)
    jv = (oracle.forward(xd + eps * v, idx, w, wgu, wd) - oracle.forward(xd - eps * v, idx, w, wgu, wd)) / (2 * eps)
    lhs = np.sum(go * jv)
    rhs = np.sum(oracle.dgrad(x, go, idx, w, wgu, wd) * v)
    assert abs(lhs - rhs) <= 1e-7 * abs(rhs) + 1e-9


# -------------------------------------------------------------- routing gradient

def _weights_from_logits(l, idx, renorm):
    """fp64 routing weights at fixed indices: softmax over all E at idx, or over the selected."""
    l = np.asarray(l, np.float64)
    if renorm:
        sel = np.take_along_axis(l, idx, 1)
        ex = np.exp(sel - sel.max(1, keepdims=True))
        return ex / ex.sum(1, keepdims=True)
    ex = np.exp(l - l.max(1, keepdims=True))
    return np.take_along_axis(ex / ex.sum(1, keepdims=True), idx, 1)


@pytest.mark.parametrize("renorm", [True, False])
def test_router_grad_dw_matches_central_finite_differences(renorm):
    """dL/dw by differencing L(w) = <grad_out, y(w)> (y is linear in w)."""
    x, idx, w, wgu, wd, *_ = _tiny_problem(E=5, H=64, I=64, T=6, k=2, seed=21, renorm=renorm)
    go = np.random.default_rng(22).standard_normal(x.shape)
    dw, _ = oracle.router_grad(x, go, None, idx, renorm, wgu, wd)
    eps = 1e-3
    num = np.zeros_like(dw)
    for t in range(x.shape[0]):
        for j in range(idx.shape[1]):
            wp, wm = w.copy(), w.copy()
            wp[t, j] += eps
            wm[t, j] -= eps
            num[t, j] = ((oracle.forward(x, idx, wp, wgu, wd) - oracle.forward(x, idx, wm, wgu, wd)) * go).sum() / (2 * eps)
    np.testing.assert_allclose(dw, num, rtol=1e-8, atol=1e-10 * np.abs(num).max())


@pytest.mark.parametrize("renorm", [True, False])
def test_router_grad_logits_match_central_finite_differences(renorm):
    """dL/dlogits by differencing L(l) = <grad_out, y(w(l))> with the indices held."""
    rng = np.random.default_rng(31)
    E, H, I, T, k = 6, 64, 64, 5, 3
    x, _, _, wgu, wd, *_ = _tiny_problem(E=E, H=H, I=I, T=T, k=k, seed=32)
    l = rng.standard_normal((T, E)).astype(np.float32)
    idx, w = oracle.route(l, k, renorm)
    np.testing.assert_allclose(_weights_from_logits(l, idx, renorm), w, rtol=1e-12)
    go = rng.standard_normal(x.shape)
    _, dl = oracle.router_grad(x, go, l, idx, renorm, wgu, wd)
    eps = 1e-4
    num = np.zeros((T, E))
    l64 = l.astype(np.float64)
    for t in range(T):
        for e in range(E):
            lp, lm = l64.copy(), l64.copy()
            lp[t, e] += eps
            lm[t, e] -= eps
            fp = (oracle.forward(x, idx, _weights_from_logits(lp, idx, renorm), wgu, wd) * go).sum()
            fm = (oracle.forward(x, idx, _weights_from_logits(lm, idx, renorm), wgu, wd) * go).sum()
            num[t, e] = (fp - fm) / (2 * eps)
    np.testing.assert_allclose(dl, num, rtol=1e-6, atol=1e-7 * np.abs(num).max())
    if renorm:   # logits outside the top-k do not move renormalised weights
        for t in range(T):
            assert np.all(np.delete(dl[t], idx[t]) == 0.0)


@pytest.mark.parametrize("renorm", [True, False])
def test_router_grad_logits_sum_to_zero_and_k1_renorm_is_zero(renorm):
    """Softmax gradients sum to zero over the logits; with k = 1 and renormalisation the
    weight is the constant 1, so the logit gradient vanishes."""
    rng = np.random.default_rng(41)
    x, _, _, wgu, wd, *_ = _tiny_problem(E=7, H=64, I=64, T=9, k=2, seed=42)
    l = rng.standard_normal((9, 7)).astype(np.float32)
    go = rng.standard_normal(x.shape)
    idx, _ = oracle.route(l, 2, renorm)
    _, dl = oracle.router_grad(x, go, l, idx, renorm, wgu, wd)
    assert np.abs(dl.sum(1)).max() <= 1e-12 * np.abs(dl).max()
    idx1, _ = oracle.route(l, 1, True)
    _, dl1 = oracle.router_grad(x, go, l, idx1, True, wgu, wd)
    assert np.all(dl1 == 0.0)


# ------------------------------------------------------ seeded workloads

def test_zipf_router_hot_set():
    """The Qwen3-shaped router bias puts about half the selections on ~6% of experts."""
    w = wl.QWEN3
    x = wl.activations(w)
    l = wl.router_logits(w, x).numpy()
    idx, _ = oracle.route(l, w.k, w.renorm)
    c = np.sort(np.bincount(idx.ravel(), minlength=w.E))[::-1]
    share = c[:8].sum() / c.sum()
    assert 0.35 < share < 0.65


# -------------------------------------------------------------- gpt-oss expert variant
# Clamped GLU h = (u' + 1) g' sigmoid(alpha g'), g' = min(g, L), u' = clamp(u, -L, L),
# with per-expert biases on g, u (bgu [E, 2I], gate half first) and on the down output.

GLU = oracle.ACT_CLAMPED_GLU


def _biases(E, H, I, seed, scale=0.5):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((E, 2 * I)) * scale).astype(np.float32), \
        (rng.standard_normal((E, H)) * scale).astype(np.float32)


def test_clamped_glu_alpha1_unclamped_is_swiglu_with_unit_up_bias():
    """alpha = 1, L = inf: (u + 1) silu(g) is SwiGLU with the up pre-activation
    shifted by one, i.e. SwiGLU with up bias 1 (gate bias 0)."""
    x, idx, w, wgu, wd, *_ = _tiny_problem(E=5, H=64, I=64, T=12, k=2, seed=31)
    E, I2, H = wgu.shape
    bgu1 = np.concatenate([np.zeros((E, I2 // 2)), np.ones((E, I2 // 2))], 1).astype(np.float32)
    y_glu = oracle.forward(x, idx, w, wgu, wd, act=GLU, alpha=1.0, limit=np.inf)
    y_sw = oracle.forward(x, idx, w, wgu, wd, bgu=bgu1)
    np.testing.assert_allclose(y_glu, y_sw, rtol=1e-12, atol=1e-14 * np.abs(y_sw).max())


def test_clamped_glu_large_alpha_is_relu_gated():
    """alpha -> inf turns sigmoid(alpha g) into the unit step: h -> (u' + 1) relu(g')."""
    x, idx, w, wgu, wd, *_ = _tiny_problem(E=4, H=64, I=64, T=10, k=2, seed=32)
    E, I2, H = wgu.shape
    I = I2 // 2
    y = oracle.forward(x, idx, w, wgu, wd, act=GLU, alpha=1e9, limit=0.3)
    xd = x.astype(np.float64)
    ref = np.zeros_like(y)
    for t in range(x.shape[0]):
        for j in range(idx.shape[1]):
            e = idx[t, j]
            g = wgu[e, :I].astype(np.float64) @ xd[t]
            u = wgu[e, I:].astype(np.float64) @ xd[t]
            h = (np.clip(u, -0.3, 0.3) + 1.0) * np.maximum(np.minimum(g, 0.3), 0.0)
            ref[t] += w[t, j] * (wd[e].astype(np.float64) @ h)
    np.testing.assert_allclose(y, ref, rtol=1e-9, atol=1e-12 * np.abs(ref).max())


def test_clamped_glu_clamp_invariances():
    """Outside the clamp the up pre-activation does not matter; inside it the limit does not."""
    x, idx, w, wgu, wd, *_ = _tiny_problem(E=4, H=64, I=64, T=9, k=2, seed=33)
    E, I2, H = wgu.shape
    I = I2 // 2
    # every |g|, |u| below 10: a limit of 10 equals no limit
    np.testing.assert_allclose(oracle.forward(x, idx, w, wgu, wd, act=GLU, limit=10.0),
                               oracle.forward(x, idx, w, wgu, wd, act=GLU, limit=np.inf), rtol=0, atol=0)
    # up bias 5 pushes every u above L = 1: scaling the up weights changes nothing
    b = np.concatenate([np.zeros((E, I)), np.full((E, I), 5.0)], 1).astype(np.float32)
    w2 = wgu.copy()
    w2[:, I:] *= 0.5
    y1 = oracle.forward(x, idx, w, wgu, wd, act=GLU, limit=1.0, bgu=b)
    y2 = oracle.forward(x, idx, w, w2, wd, act=GLU, limit=1.0, bgu=b)
    np.testing.assert_array_equal(y1, y2)


def test_down_bias_adds_routing_weighted_bias():
    """y(bd) - y(0) = sum_j w_{t,j} bd[e_{t,j}] for every token."""
    x, idx, w, wgu, wd, *_ = _tiny_problem(E=6, H=64, I=64, T=11, k=3, seed=34)
    E, I2, H = wgu.shape
    bgu, bd = _biases(E, H, I2 // 2, 35)
    d = oracle.forward(x, idx, w, wgu, wd, act=GLU, bgu=bgu, bd=bd) - oracle.forward(x, idx, w, wgu, wd, act=GLU,
                                                                                      bgu=bgu)
    ref = np.einsum("tj,tjh->th", w, bd[idx].astype(np.float64))
    np.testing.assert_allclose(d, ref, rtol=1e-10, atol=1e-12)


def test_clamped_glu_dgrad_matches_central_finite_differences():
    """Biases and a limit that clamps part of g and u (no pre-activation within eps of a kink)."""
    x, idx, w, wgu, wd, *_ = _tiny_problem(E=4, H=64, I=64, T=6, k=2, seed=36)
    E, I2, H = wgu.shape
    bgu, bd = _biases(E, H, I2 // 2, 37)
    kw = dict(act=GLU, alpha=1.702, limit=0.8, bgu=bgu)
    go = np.random.default_rng(38).standard_normal(x.shape)
    gx = oracle.dgrad(x, go, idx, w, wgu, wd, **kw)
    eps = 1e-6
    num = np.zeros_like(gx)
    for t in range(x.shape[0]):
        for c in range(x.shape[1]):
            xp = x.astype(np.float64).copy()
            xm = xp.copy()
            xp[t, c] += eps
            xm[t, c] -= eps
            fp = (oracle.forward(xp, idx, w, wgu, wd, tokens=[t], bd=bd, **kw) * go[t]).sum()
            fm = (oracle.forward(xm, idx, w, wgu, wd, tokens=[t], bd=bd, **kw) * go[t]).sum()
            num[t, c] = (fp - fm) / (2 * eps)
    np.testing.assert_allclose(gx, num, rtol=1e-6, atol=1e-6 * np.abs(num).max())
    # the clamp is active somewhere, so the test exercises the zero-gradient branch
    xd = x.astype(np.float64)
    g = np.einsum("th,eih->eti", xd, wgu[:, :I2 // 2]) + bgu[:, None, :I2 // 2]
    u = np.einsum("th,eih->eti", xd, wgu[:, I2 // 2:]) + bgu[:, None, I2 // 2:]
    assert (g > 0.8).any() and (np.abs(u) > 0.8).any()


def test_clamped_glu_router_grad_dw_matches_central_finite_differences():
    x, idx, w, wgu, wd, *_ = _tiny_problem(E=5, H=64, I=64, T=6, k=2, seed=39)
    E, I2, H = wgu.shape
    bgu, bd = _biases(E, H, I2 // 2, 40)
    kw = dict(act=GLU, alpha=1.702, limit=0.8, bgu=bgu, bd=bd)
    go = np.random.default_rng(41).standard_normal(x.shape)
    dw, _ = oracle.router_grad(x, go, None, idx, True, wgu, wd, **kw)
    eps = 1e-3
    num = np.zeros_like(dw)
    for t in range(x.shape[0]):
        for j in range(idx.shape[1]):
            wp, wm = w.copy(), w.copy()
            wp[t, j] += eps
            wm[t, j] -= eps
            num[t, j] = ((oracle.forward(x, idx, wp, wgu, wd, **kw) - oracle.forward(x, idx, wm, wgu, wd, **kw))
                         * go).sum() / (2 * eps)
    np.testing.assert_allclose(dw, num, rtol=1e-8, atol=1e-10 * np.abs(num).max())


# -------------------------------------------------------------- per-expert LoRA (next row)
# Adapters A_gu [E,r,H], B_gu [E,2I,r], A_d [E,r,I], B_d [E,H,r]; update scale s = alpha / r.

def _adapters(E, H, I, r, seed, zero_b=False):
    rng = np.random.default_rng(seed)
    agu = (rng.standard_normal((E, r, H)) * 0.1).astype(np.float32)
    bgu_l = np.zeros((E, 2 * I, r), np.float32) if zero_b else (rng.standard_normal((E, 2 * I, r)) * 0.1).astype(np.float32)
    ad = (rng.standard_normal((E, r, I)) * 0.1).astype(np.float32)
    bd_l = np.zeros((E, H, r), np.float32) if zero_b else (rng.standard_normal((E, H, r)) * 0.1).astype(np.float32)
    return agu, bgu_l, ad, bd_l


@pytest.mark.parametrize("act", [oracle.ACT_SWIGLU, GLU])
def test_lora_zero_b_is_the_base_layer(act):
    """LoRA's B starts at zero: the adapted layer is then exactly the base layer."""
    x, idx, w, wgu, wd, *_ = _tiny_problem(E=5, H=64, I=64, T=10, k=2, seed=81)
    ad_ = _adapters(5, 64, 64, 8, 82, zero_b=True)
    bgu, bd = _biases(5, 64, 64, 83)
    np.testing.assert_array_equal(oracle.lora_forward(x, idx, w, wgu, wd, *ad_, 2.0, act=act, bgu=bgu, bd=bd),
                                  oracle.forward(x, idx, w, wgu, wd, act=act, bgu=bgu, bd=bd))


def test_lora_equals_base_with_merged_weights():
    """x W^T + s (x A^T) B^T = x (W + s B A)^T: the adapted layer equals the base layer
    evaluated with the merged dense weights."""
    x, idx, w, wgu, wd, *_ = _tiny_problem(E=4, H=64, I=64, T=12, k=2, seed=84)
    agu, bgu_l, ad, bd_l = _adapters(4, 64, 64, 4, 85)
    s = 16.0 / 4
    mg = (wgu.astype(np.float64) + s * np.einsum("eor,erh->eoh", bgu_l, agu)).astype(np.float32)
    md = (wd.astype(np.float64) + s * np.einsum("ehr,eri->ehi", bd_l, ad)).astype(np.float32)
    y = oracle.lora_forward(x, idx, w, wgu, wd, agu, bgu_l, ad, bd_l, s)
    ref = oracle.forward(x, idx, w, mg, md)
    np.testing.assert_allclose(y, ref, rtol=2e-5, atol=2e-6 * np.abs(ref).max())


@pytest.mark.parametrize("act", [oracle.ACT_SWIGLU, GLU])
def test_lora_single_expert_matches_torch_autograd(act):
    """E = 1, k = 1, w = 1: a dense MLP with LoRA on both projections; forward and every
    gradient against torch autograd in fp64."""
    E, H, I, r, T = 1, 64, 64, 4, 7
    x, _, _, wgu, wd, *_ = _tiny_problem(E=E, H=H, I=I, T=T, k=1, seed=86)
    idx = np.zeros((T, 1), np.int32)
    w = np.ones((T, 1))
    agu, bgu_l, ad, bd_l = _adapters(E, H, I, r, 87)
    bgu, bd = _biases(E, H, I, 88)
    s, al, L = 2.5, 1.702, 0.9
    go = np.random.default_rng(89).standard_normal((T, H))
    y = oracle.lora_forward(x, idx, w, wgu, wd, agu, bgu_l, ad, bd_l, s, act=act, alpha=al, limit=L, bgu=bgu, bd=bd)
    gx, dag, dbg, dad, dbd = oracle.lora_backward(x, go, idx, w, wgu, wd, agu, bgu_l, ad, bd_l, s, act=act, alpha=al,
                                                  limit=L, bgu=bgu)
    tt = lambda a, grad=False: torch.tensor(np.asarray(a, np.float64), requires_grad=grad)
    X, Ag, Bg, Ad, Bd = tt(x, True), tt(agu[0], True), tt(bgu_l[0], True), tt(ad[0], True), tt(bd_l[0], True)
    gu = X @ tt(wgu[0]).T + s * (X @ Ag.T) @ Bg.T + tt(bgu[0])
    g, u = gu[:, :I], gu[:, I:]
    if act == oracle.ACT_SWIGLU:
        h = torch.nn.functional.silu(g) * u
    else:
        gc, uc = torch.clamp(g, max=L), torch.clamp(u, -L, L)
        h = (uc + 1) * gc * torch.sigmoid(al * gc)
    Y = h @ tt(wd[0]).T + s * (h @ Ad.T) @ Bd.T + tt(bd[0])
    (Y * tt(go)).sum().backward()
    np.testing.assert_allclose(y, Y.detach().numpy(), rtol=1e-11, atol=1e-13)
    for mine, ref in ((gx, X.grad), (dag[0], Ag.grad), (dbg[0], Bg.grad), (dad[0], Ad.grad), (dbd[0], Bd.grad)):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=1e-10, atol=1e-12 * np.abs(ref.numpy()).max())


def test_lora_routed_gradients_match_central_finite_differences():
    """Several experts, k = 2, routing weights: the adapter gradients sum over each
    expert's pairs (sampled entries) and grad_x (all entries) by central differences."""
    E, H, I, r = 4, 64, 64, 4
    x, idx, w, wgu, wd, *_ = _tiny_problem(E=E, H=H, I=I, T=6, k=2, seed=90)
    ad_ = list(_adapters(E, H, I, r, 91))
    s = 4.0
    go = np.random.default_rng(92).standard_normal(x.shape)
    grads = oracle.lora_backward(x, go, idx, w, wgu, wd, *ad_, s)
    L = lambda xx, aa: (oracle.lora_forward(xx, idx, w, wgu, wd, *aa, s) * go).sum()
    eps = 1e-6
    xd = x.astype(np.float64)
    num = np.zeros_like(xd)
    for t in range(x.shape[0]):
        for c in range(0, H, 5):
            xp, xm = xd.copy(), xd.copy()
            xp[t, c] += eps
            xm[t, c] -= eps
            num[t, c] = (L(xp, ad_) - L(xm, ad_)) / (2 * eps)
    sel = np.zeros_like(xd, bool)
    sel[:, 0:H:5] = True
    np.testing.assert_allclose(grads[0][sel], num[sel], rtol=1e-6, atol=1e-6 * np.abs(num).max())
    rng = np.random.default_rng(93)
    for which in range(4):
        g_an = grads[1 + which]
        for _ in range(12):
            pos = tuple(int(rng.integers(0, n)) for n in ad_[which].shape)
            eps_w = 1e-3   # the adapters are fp32 inputs: perturb by a representable step
            ap, am = [a.copy() for a in ad_], [a.copy() for a in ad_]
            ap[which][pos] += eps_w
            am[which][pos] -= eps_w
            d = (ap[which][pos] - am[which][pos])   # the exact fp32 step taken
            num_w = (L(xd, ap) - L(xd, am)) / d
            assert abs(num_w - g_an[pos]) <= 1e-5 * max(1.0, abs(g_an[pos])), (which, pos, num_w, g_an[pos])
