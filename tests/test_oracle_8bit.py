"""Pins for the oracle's 8-bit blockwise modes (int8: the dynamic tree map;
fp8: the E4M3 grid over 448), checked against torch's float8_e4m3fn decoding,
the structure the dynamic map's definition fixes, brute force, and the support
matrix's reconstruction-error ordering int8 < fp8 < nf4 < fp4.  CPU only."""
import numpy as np
import pytest
import torch

import oracle


def test_fp8_codebook_is_torch_e4m3_over_448():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).float().numpy().astype(np.float64) / 448.0
    got = oracle.codebook8(oracle.FP8).astype(np.float64)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok].astype(np.float32).astype(np.float64))
    assert np.nanmax(got) == 1.0 and np.nanmin(got) == -1.0


def test_int8_dynamic_map_structure():
    """Decimal exponent bands: tail codes with E leading zeros hold 2^(6-E) values
    in 10^-E * [0.1, 1], increasing with the fraction bits; the sign bit negates;
    tail 0 is 0 and, with the sign set, the endpoint +1; 256 distinct values."""
    v = oracle.codebook8(oracle.INT8).astype(np.float64)
    assert v[0] == 0.0 and v[128] == 1.0
    assert len(np.unique(v)) == 256
    for t in range(1, 128):
        assert v[128 | t] == -v[t]
        E = 7 - t.bit_length()
        band = [c for c in range(1, 128) if 7 - c.bit_length() == E]
        assert len(band) == 2 ** (6 - E)
        assert 10.0 ** -E * 0.1 < v[t] < 10.0 ** -E
    for E in range(7):
        band = [c for c in range(1, 128) if 7 - c.bit_length() == E]
        assert np.all(np.diff(v[band]) > 0)   # the fraction bits count upward
        # equal bins on [0.1, 1]: consecutive centres 0.9 / 2^F * 10^-E apart
        if len(band) > 1:
            assert np.allclose(np.diff(v[band]), 0.9 / len(band) * 10.0 ** -E, rtol=1e-5)


@pytest.mark.parametrize("cb", [oracle.INT8, oracle.FP8])
def test_brute_force_nearest_tie_rule_and_round_trip(cb):
    """Every code is the nearest value (brute force over the table; an exact tie to
    the smaller value), so |w - deq| <= absmax * (largest gap) / 2."""
    table = oracle.codebook8(cb)
    valid = [q for q in range(256) if not np.isnan(table[q]) and not (cb == oracle.FP8 and q == 0x80)]
    vals = np.array([table[q] for q in valid], np.float64)
    rng = np.random.default_rng(5)
    w = (rng.standard_normal((2, 4, 128)) * 0.02).astype(np.float32)
    codes, absmax = oracle.quantize8(w, cb)
    for blk in range(absmax.size):
        a = absmax.reshape(-1)[blk]
        for i in range(64):
            x = w.reshape(-1)[blk * 64 + i]
            n = np.float32(x) / np.float32(a)
            d = np.abs(vals - n)
            best = np.flatnonzero(d == d.min())
            want = vals[best].min()   # a tie goes to the smaller value
            assert table[codes.reshape(-1)[blk * 64 + i]] == np.float32(want)
    srt = np.sort(vals)
    gap = np.diff(srt).max()
    deq = oracle.dequantize8(codes, absmax, w.shape, cb, "f32")
    bound = absmax.reshape(2, 4, 2, 1).repeat(64, 3).reshape(w.shape) * gap / 2
    assert np.all(np.abs(deq - w) <= bound * (1 + 1e-5))   # fp32 rounding of table and products


@pytest.mark.parametrize("cb", [oracle.INT8, oracle.FP8])
def test_exact_reproduction_idempotence_and_zero_block(cb):
    table = oracle.codebook8(cb)
    valid = [q for q in range(256) if not np.isnan(table[q]) and not (cb == oracle.FP8 and q == 0x80)]
    rng = np.random.default_rng(6)
    pick = rng.choice(valid, size=63, replace=False)
    blk = np.concatenate([[1.0], table[pick]]).astype(np.float32)   # absmax 1: values reproduce exactly
    w = np.stack([blk, np.zeros(64, np.float32)]).reshape(1, 2, 64)
    codes, absmax = oracle.quantize8(w, cb)
    assert absmax[0, 0] == 1.0 and absmax[0, 1] == 0.0
    got = oracle.dequantize8(codes, absmax, w.shape, cb, "f32")
    assert np.array_equal(got, w)
    c2, a2 = oracle.quantize8(oracle.dequantize8(codes, absmax, w.shape, cb, "f32"), cb)
    assert np.array_equal(c2, codes) and np.array_equal(a2, absmax)


def test_support_matrix_error_ordering():
    """On N(0, 0.02) blocks: int8 < fp8 < nf4 < fp4 reconstruction error ([P1]
    "Storage modes: the support matrix")."""
    rng = np.random.default_rng(7)
    w = (rng.standard_normal((4, 128, 512)) * 0.02).astype(np.float32)
    err = {}
    for name, cb in (("int8", oracle.INT8), ("fp8", oracle.FP8)):
        c, a = oracle.quantize8(w, cb)
        err[name] = np.sqrt(np.mean((oracle.dequantize8(c, a, w.shape, cb, "f32") - w) ** 2) / np.mean(w ** 2))
    for name, cb in (("nf4", oracle.NF4), ("fp4", oracle.FP4)):
        p, a = oracle.quantize(w, cb)
        err[name] = np.sqrt(np.mean((oracle.dequantize(p, a, w.shape, cb, "f32") - w) ** 2) / np.mean(w ** 2))
    assert err["int8"] < err["fp8"] < err["nf4"] < err["fp4"], err
