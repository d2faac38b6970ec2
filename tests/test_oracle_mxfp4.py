"""Pins for the oracle's MXFP4 quantize / dequantize (OCP Microscaling Formats
v1.0: 32-element blocks, an E8M0 scale 2^X stored as X + 127, E2M1 elements).
Each test checks the oracle against something other than itself: values
built by hand from the format's definition, numpy's log2 for the scale
exponent, a brute-force nearest-value search, the spec's round-trip bound.
CPU only."""
import numpy as np
import pytest

import oracle

E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _q(w):
    w = np.asarray(w, np.float32)
    return oracle.quantize_mxfp4(w.reshape(1, 1, -1))


def _codes(packed):
    hi, lo = packed.reshape(-1) >> 4, packed.reshape(-1) & 15
    return np.stack([hi, lo], 1).reshape(-1)


def _value(code, X):
    m = E2M1[code & 7]
    return (-m if code & 8 else m) * 2.0 ** X


@pytest.mark.parametrize("X", [-20, -3, 0, 5])
def test_exact_reproduction_of_scaled_e2m1_values(X):
    """A block holding every E2M1 value times 2^X (both signs) keeps its scale and
    its codes, and dequantizes to exactly those values."""
    vals = np.concatenate([E2M1, -E2M1[1:], E2M1[:8], -E2M1[1:8], [6.0, -6.0]])[:32] * 2.0 ** X
    packed, scales = _q(vals)
    assert scales[0, 0, 0] == X + 127
    codes = _codes(packed)
    want = [int(np.argmax(E2M1 == abs(v) / 2.0 ** X)) | (8 if v < 0 else 0) for v in vals]
    assert list(codes) == want
    back = oracle.dequantize_mxfp4(packed, scales, (1, 1, 32), "f32").reshape(-1)
    assert np.array_equal(back, vals.astype(np.float32))
    bf = oracle.dequantize_mxfp4(packed, scales, (1, 1, 32)).reshape(-1)
    assert np.array_equal(bf, vals.astype(np.float32))   # exactly representable in bf16


def test_scale_exponent_is_floor_log2_amax_minus_two():
    """X = floor(log2(max|v|)) - 2, from numpy's float64 log2, over maxima spread
    across many binades and exactly at powers of two; clamped at -127."""
    rng = np.random.default_rng(1)
    amax = np.concatenate([2.0 ** rng.uniform(-60, 60, 200), 2.0 ** np.arange(-40, 40), [6.0, 7.999, 8.0, 0.75]])
    for a in amax.astype(np.float32):
        block = np.zeros(32, np.float32)
        block[7] = -a
        block[3] = a / 3
        _, scales = _q(block)
        X = int(np.floor(np.log2(np.float64(a)))) - 2
        assert scales[0, 0, 0] == max(X, -127) + 127, a
    _, scales = _q(np.full(32, 1e-40, np.float32))   # floor(log2) = -133: clamped
    assert scales[0, 0, 0] == 0


def test_ties_to_even_and_saturation():
    """Midpoints between E2M1 values round to the even code (0, 1, 2, 4); values
    between 6 and 8 times the scale saturate at 6.  amax = 7.5 gives X = 0."""
    p = [7.5, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.9, -0.75, -5.0, 0.24, 0.26]
    want = [6.0, 0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 6.0, -1.0, -4.0, 0.0, 0.5]
    block = np.zeros(32, np.float32)
    block[:len(p)] = p
    packed, scales = _q(block)
    assert scales[0, 0, 0] == 127
    back = oracle.dequantize_mxfp4(packed, scales, (1, 1, 32), "f32").reshape(-1)
    assert list(back[:len(p)]) == want


def test_brute_force_nearest_and_round_trip_bound():
    """Every element equals the brute-force nearest of the 15 signed E2M1 values
    times 2^X (ties to the even code, saturating), so |w - deq| <= 2^X where
    |w| <= 6 * 2^X and < 2^(X+1) above it."""
    rng = np.random.default_rng(2)
    w = (rng.standard_normal((3, 5, 128)) * 0.02).astype(np.float32)
    w[0, 0, :32] *= 1e-3
    packed, scales = oracle.quantize_mxfp4(w)
    back = oracle.dequantize_mxfp4(packed, scales, w.shape, "f32")
    cand = np.concatenate([E2M1, -E2M1[1:]])
    cand_code = np.concatenate([np.arange(8), 8 + np.arange(1, 8)])
    for e in range(3):
        for o in range(5):
            for j in range(4):
                blk = w[e, o, 32 * j:32 * j + 32].astype(np.float64)
                X = int(scales[e, o, j]) - 127
                for i, v in enumerate(blk):
                    p = v / 2.0 ** X
                    d = np.abs(cand - min(max(p, -6.0), 6.0))
                    best = np.flatnonzero(d == d.min())
                    if len(best) > 1:   # a tie: the even E2M1 code
                        best = [b for b in best if (cand_code[b] & 1) == 0]
                    want = cand[best[0]] * 2.0 ** X
                    got = back[e, o, 32 * j + i]
                    assert got == np.float32(want), (e, o, j, i, p)
                    bound = 2.0 ** X if abs(p) <= 6 else 2.0 ** (X + 1)
                    assert abs(got - v) <= bound


def test_idempotent_zero_block_padding_and_layout():
    rng = np.random.default_rng(3)
    w = (rng.standard_normal((2, 3, 96)) * 0.05).astype(np.float32)
    w[1, 2, 32:64] = 0.0
    p1, s1 = oracle.quantize_mxfp4(w)
    p2, s2 = oracle.quantize_mxfp4(oracle.dequantize_mxfp4(p1, s1, w.shape, "f32"))
    assert np.array_equal(p1, p2) and np.array_equal(s1, s2)
    assert s1.shape == (2, 3, 16) and np.all(s1[:, :, 3:] == 0)      # 96/32 = 3 scales, rows padded to 16
    assert s1[1, 2, 1] == 0 and np.all(p1[1].reshape(3, 48)[2, 16:32] == 0)   # all-zero block: X = -127, +0
    blk = np.zeros(32, np.float32)
    blk[0], blk[1] = 1.0, -0.5            # amax 1 -> X = -2: 1.0 / 0.25 = 4 (code 6), -0.5 / 0.25 = -2 (code 8|4)
    packed, _ = _q(blk)
    assert packed.reshape(-1)[0] == (6 << 4) | (8 | 4)   # first element in the high nibble
    with pytest.raises(RuntimeError):
        oracle.quantize_mxfp4(np.zeros((1, 1, 48), np.float32))


def test_mxfp4_error_vs_absmax_fp4_on_gaussian_weights():
    """On N(0, 0.02) blocks the power-of-two 32-element scales reconstruct within
    the same range as the 64-element absmax FP4 codebook (both E2M1 grids):
    rel-RMSE between 0.05 and 0.2 each, recorded for the storage comparison."""
    rng = np.random.default_rng(4)
    w = (rng.standard_normal((4, 256, 256)) * 0.02).astype(np.float32)
    pm, sm = oracle.quantize_mxfp4(w)
    dm = oracle.dequantize_mxfp4(pm, sm, w.shape, "f32")
    pf, af = oracle.quantize(w, oracle.FP4)
    df = oracle.dequantize(pf, af, w.shape, oracle.FP4, "f32")
    rm = np.sqrt(np.mean((dm - w) ** 2) / np.mean(w ** 2))
    rf = np.sqrt(np.mean((df - w) ** 2) / np.mean(w ** 2))
    assert 0.05 < rm < 0.2 and 0.05 < rf < 0.2, (rm, rf)
