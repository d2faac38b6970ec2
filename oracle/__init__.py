"""CPU oracle for the NF4 Mixture-of-Experts expert path.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package.  The product library never
does, and the two share no code.

The arithmetic lives in ``e4b_oracle.c``: a plain C statement of quantize,
dequantize, routing, grouping, forward and input gradient, each function citing
the page section it follows.  This module only compiles that file with gcc and
marshals numpy arrays through ctypes.

Parity status of each function (what pins it is in ``tests/test_oracle_pins.py``):
  quantize / dequantize  pinned (round-trip bound, exact reproduction, idempotence,
                         tie rule, validation, NF4 < FP4 error ordering, codebook vs
                         the NormalFloat quantile construction)
  route / permute        pinned (brute-force sort, softmax ratio closed form, bijection)
  forward                pinned (fp64 dense all-experts reference; E=1 dense SwiGLU MLP)
  dgrad                  pinned (central finite differences; adjoint identity)
  int8 / fp8 quantize / dequantize
                         pinned (fp8 values vs torch's float8_e4m3fn decoding, int8 map
                         structure from its definition, exact reproduction, tie rule,
                         idempotence, round-trip bound, the support matrix's error
                         ordering int8 < fp8 < nf4 < fp4); parity with bitsandbytes'
                         own tables unpinned (not on the pages)
  MXFP4 quantize / dequantize
                         pinned (exact reproduction of scaled E2M1 values, the scale
                         exponent on hand-picked maxima and its clamp, ties to even,
                         saturation, round-trip bound, idempotence, padding)
  FP4 codebook vs bitsandbytes' own fp4 table: parity unpinned (not on the pages).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "e4b_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libe4b_oracle.so")
_lock = threading.Lock()
_lib = None

NF4, FP4 = 0, 1
INT8, FP8 = 3, 4      # 8-bit blockwise codebooks (one byte per element)


def build(force: bool = False) -> str:
    """Compile the oracle into a shared library beside its source."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _L():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            P = ctypes.c_void_p
            i64, i32 = ctypes.c_int64, ctypes.c_int
            lib.e4bo_quantize.argtypes = [P, i64, i64, i64, i32, i32, P, P]
            lib.e4bo_dequantize_f32.argtypes = [P, P, i64, i32, i32, P]
            lib.e4bo_dequantize_bf16.argtypes = [P, P, i64, i32, i32, P]
            lib.e4bo_quantize_mxfp4.argtypes = [P, i64, i64, i64, P, P]
            lib.e4bo_quantize8.argtypes = [P, i64, i64, i64, i32, P, P]
            lib.e4bo_dequantize8.argtypes = [P, P, i64, i32, i32, P]
            lib.e4bo_codebook8.argtypes = [i32, P]
            lib.e4bo_dequantize_mxfp4.argtypes = [P, P, i64, i64, i64, i32, P]
            lib.e4bo_mxfp4_scale_stride.argtypes = [i64]
            lib.e4bo_mxfp4_scale_stride.restype = i64
            lib.e4bo_route.argtypes = [P, i64, i32, i32, i32, P, P]
            lib.e4bo_permute.argtypes = [P, i64, i32, i32, P, P, P]
            dbl = ctypes.c_double
            lib.e4bo_forward.argtypes = [P, i64, i32, i32, i32, i32, P, P, P, P, P, i64, i32, dbl, dbl, P, P, P]
            lib.e4bo_dgrad.argtypes = [P, P, i64, i32, i32, i32, i32, P, P, P, P, P, i64, i32, dbl, dbl, P, P]
            lib.e4bo_router_grad.argtypes = [P, P, P, i64, i32, i32, i32, i32, i32, P, P, P, P, i64, i32, dbl, dbl,
                                             P, P, P, P]
            lib.e4bo_lora_forward.argtypes = [P, i64, i32, i32, i32, i32, P, P, P, P, P, P, P, P, i32, dbl, i32, dbl,
                                              dbl, P, P, P]
            lib.e4bo_lora_backward.argtypes = [P, P, i64, i32, i32, i32, i32, P, P, P, P, P, P, P, P, i32, dbl, i32,
                                               dbl, dbl, P, P, P, P, P, P]
            lib.e4bo_codebook.argtypes = [i32, P]
            lib.e4bo_f32_to_bf16.argtypes = [ctypes.c_float]
            lib.e4bo_f32_to_bf16.restype = ctypes.c_uint16
            for f in ("e4bo_quantize", "e4bo_dequantize_f32", "e4bo_dequantize_bf16",
                      "e4bo_route", "e4bo_permute", "e4bo_forward", "e4bo_dgrad", "e4bo_router_grad"):
                getattr(lib, f).restype = ctypes.c_int
            lib.e4bo_num_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


class OracleError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned status {code}")
        self.code = code


def _check(fn: str, rc: int):
    if rc != 0:
        raise OracleError(fn, rc)


def num_threads() -> int:
    return int(_L().e4bo_num_threads())


def codebook(cb: int = NF4) -> np.ndarray:
    out = np.zeros(16, np.float32)
    _L().e4bo_codebook(cb, _p(out))
    return out


def f32_to_bf16_bits(values: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest-even); returns the uint16 bit patterns."""
    lib = _L()
    v = np.ascontiguousarray(values, np.float32).ravel()
    return np.array([lib.e4bo_f32_to_bf16(float(f)) for f in v], np.uint16).reshape(np.shape(values))


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def quantize(w: np.ndarray, cb: int = NF4, blocksize: int = 64):
    """w: fp32 [E, out, in] -> (packed uint8 [E, out*in/2], absmax fp32 [E, out*in/64])."""
    w = np.ascontiguousarray(w, np.float32)
    if w.ndim != 3:
        raise ValueError("quantize expects a 3-D [E, out, in] stack")
    E, o, i = w.shape
    packed = np.zeros((E, o * i // 2), np.uint8)
    absmax = np.zeros((E, max(o * i // max(blocksize, 1), 0)), np.float32)
    _check("e4bo_quantize", _L().e4bo_quantize(_p(w), E, o, i, blocksize, cb, _p(packed), _p(absmax)))
    return packed, absmax


def dequantize(packed: np.ndarray, absmax: np.ndarray, shape, cb: int = NF4,
               out_dtype: str = "bf16", blocksize: int = 64) -> np.ndarray:
    """Packed bytes + absmax -> [E, out, in] values.  out_dtype 'bf16' returns the
    bf16 values widened to fp32 (exact); 'bf16_bits' the raw uint16 patterns;
    'f32' the unrounded fp32 products."""
    packed = np.ascontiguousarray(packed, np.uint8)
    absmax = np.ascontiguousarray(absmax, np.float32)
    n = int(np.prod(shape))
    if out_dtype == "f32":
        out = np.zeros(n, np.float32)
        _check("e4bo_dequantize_f32", _L().e4bo_dequantize_f32(_p(packed), _p(absmax), n, blocksize, cb, _p(out)))
        return out.reshape(shape)
    bits = np.zeros(n, np.uint16)
    _check("e4bo_dequantize_bf16", _L().e4bo_dequantize_bf16(_p(packed), _p(absmax), n, blocksize, cb, _p(bits)))
    bits = bits.reshape(shape)
    return bits if out_dtype == "bf16_bits" else bf16_bits_to_f32(bits)


def codebook8(cb: int) -> np.ndarray:
    """The 256 values of an 8-bit codebook (INT8 or FP8), indexed by code (NaN
    for the FP8 NaN patterns)."""
    out = np.zeros(256, np.float32)
    _L().e4bo_codebook8(cb, _p(out))
    return out


def quantize8(w: np.ndarray, cb: int):
    """w: fp32 [E, out, in] -> (codes uint8 [E, out*in], absmax fp32 [E, out*in/64])."""
    w = np.ascontiguousarray(w, np.float32)
    E, o, i = w.shape
    codes = np.zeros((E, o * i), np.uint8)
    absmax = np.zeros((E, o * i // 64), np.float32)
    _check("e4bo_quantize8", _L().e4bo_quantize8(_p(w), E, o, i, cb, _p(codes), _p(absmax)))
    return codes, absmax


def dequantize8(codes: np.ndarray, absmax: np.ndarray, shape, cb: int, out_dtype: str = "bf16") -> np.ndarray:
    codes = np.ascontiguousarray(codes, np.uint8)
    absmax = np.ascontiguousarray(absmax, np.float32)
    n = int(np.prod(shape))
    if out_dtype == "f32":
        out = np.zeros(n, np.float32)
        _check("e4bo_dequantize8", _L().e4bo_dequantize8(_p(codes), _p(absmax), n, cb, 0, _p(out)))
        return out.reshape(shape)
    bits = np.zeros(n, np.uint16)
    _check("e4bo_dequantize8", _L().e4bo_dequantize8(_p(codes), _p(absmax), n, cb, 1, _p(bits)))
    bits = bits.reshape(shape)
    return bits if out_dtype == "bf16_bits" else bf16_bits_to_f32(bits)


def mxfp4_scale_stride(cols: int) -> int:
    """Bytes per row of an MXFP4 scale array: cols/32 rounded up to a multiple of 16."""
    return int(_L().e4bo_mxfp4_scale_stride(cols))


def quantize_mxfp4(w: np.ndarray):
    """w: fp32 [E, out, in] -> (packed uint8 [E, out*in/2], scales uint8 [E, out, S]),
    OCP MX v1.0 MXFP4: 32-element blocks, E8M0 scales (byte X + 127), E2M1 codes."""
    w = np.ascontiguousarray(w, np.float32)
    if w.ndim != 3:
        raise ValueError("quantize_mxfp4 expects a 3-D [E, out, in] stack")
    E, o, i = w.shape
    packed = np.zeros((E, o * i // 2), np.uint8)
    scales = np.zeros((E, o, mxfp4_scale_stride(i)), np.uint8)
    _check("e4bo_quantize_mxfp4", _L().e4bo_quantize_mxfp4(_p(w), E, o, i, _p(packed), _p(scales)))
    return packed, scales


def dequantize_mxfp4(packed: np.ndarray, scales: np.ndarray, shape, out_dtype: str = "bf16") -> np.ndarray:
    """MXFP4 packed codes + E8M0 scales -> [E, out, in]: e2m1(q) * 2^(s - 127) in fp32
    (exact), then bf16 (nearest-even; exact for these values) unless out_dtype 'f32'."""
    packed = np.ascontiguousarray(packed, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    E, o, i = shape
    if out_dtype == "f32":
        out = np.zeros(E * o * i, np.float32)
        _check("e4bo_dequantize_mxfp4", _L().e4bo_dequantize_mxfp4(_p(packed), _p(scales), E, o, i, 0, _p(out)))
        return out.reshape(shape)
    bits = np.zeros(E * o * i, np.uint16)
    _check("e4bo_dequantize_mxfp4", _L().e4bo_dequantize_mxfp4(_p(packed), _p(scales), E, o, i, 1, _p(bits)))
    bits = bits.reshape(shape)
    return bits if out_dtype == "bf16_bits" else bf16_bits_to_f32(bits)


def route(logits: np.ndarray, k: int, renorm: bool):
    """fp32 logits [T, E] -> (idx int32 [T, k], weights fp64 [T, k])."""
    logits = np.ascontiguousarray(logits, np.float32)
    T, E = logits.shape
    idx = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float64)
    _check("e4bo_route", _L().e4bo_route(_p(logits), T, E, k, int(bool(renorm)), _p(idx), _p(w)))
    return idx, w


def permute(idx: np.ndarray, E: int):
    """idx int32 [T, k] -> (counts [E], offsets [E+1], perm [T*k]) as int32."""
    idx = np.ascontiguousarray(idx, np.int32)
    T, k = idx.shape
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    perm = np.zeros(T * k, np.int32)
    _check("e4bo_permute", _L().e4bo_permute(_p(idx), T, k, E, _p(counts), _p(offsets), _p(perm)))
    return counts, offsets, perm


ACT_SWIGLU, ACT_CLAMPED_GLU = 0, 1


def _bias(b, shape):
    return None if b is None else np.ascontiguousarray(np.broadcast_to(b, shape), np.float32)


def forward(x: np.ndarray, idx: np.ndarray, w: np.ndarray, wgu: np.ndarray, wd: np.ndarray,
            tokens=None, act=ACT_SWIGLU, alpha=1.702, limit=7.0, bgu=None, bd=None) -> np.ndarray:
    """fp64 forward.  x [T,H] (any float dtype, widened to fp64), idx [T,k], w [T,k],
    wgu [E,2I,H] / wd [E,H,I] dequantized weights; act SwiGLU or the clamped GLU
    (alpha, limit); optional biases bgu [E,2I] (gate then up) and bd [E,H].  Returns
    y [nt, H] fp64 for ``tokens`` (all tokens when None)."""
    x = np.ascontiguousarray(x, np.float64)
    idx = np.ascontiguousarray(idx, np.int32)
    w = np.ascontiguousarray(w, np.float64)
    wgu = np.ascontiguousarray(wgu, np.float32)
    wd = np.ascontiguousarray(wd, np.float32)
    T, H = x.shape
    E, I2, _ = wgu.shape
    k = idx.shape[1]
    tok = None if tokens is None else np.ascontiguousarray(tokens, np.int64)
    nt = T if tok is None else tok.shape[0]
    y = np.zeros((nt, H), np.float64)
    bgu, bd = _bias(bgu, (E, I2)), _bias(bd, (E, H))
    _check("e4bo_forward", _L().e4bo_forward(_p(x), T, E, H, I2 // 2, k, _p(idx), _p(w), _p(wgu), _p(wd),
                                             None if tok is None else _p(tok), nt, int(act), float(alpha),
                                             float(limit), None if bgu is None else _p(bgu),
                                             None if bd is None else _p(bd), _p(y)))
    return y


def dgrad(x: np.ndarray, grad_out: np.ndarray, idx: np.ndarray, w: np.ndarray, wgu: np.ndarray,
          wd: np.ndarray, tokens=None, act=ACT_SWIGLU, alpha=1.702, limit=7.0, bgu=None) -> np.ndarray:
    """fp64 input gradient of the forward above with routing held constant (the
    down bias does not enter it)."""
    x = np.ascontiguousarray(x, np.float64)
    g = np.ascontiguousarray(grad_out, np.float64)
    idx = np.ascontiguousarray(idx, np.int32)
    w = np.ascontiguousarray(w, np.float64)
    wgu = np.ascontiguousarray(wgu, np.float32)
    wd = np.ascontiguousarray(wd, np.float32)
    T, H = x.shape
    E, I2, _ = wgu.shape
    k = idx.shape[1]
    tok = None if tokens is None else np.ascontiguousarray(tokens, np.int64)
    nt = T if tok is None else tok.shape[0]
    gx = np.zeros((nt, H), np.float64)
    bgu = _bias(bgu, (E, I2))
    _check("e4bo_dgrad", _L().e4bo_dgrad(_p(x), _p(g), T, E, H, I2 // 2, k, _p(idx), _p(w), _p(wgu), _p(wd),
                                         None if tok is None else _p(tok), nt, int(act), float(alpha), float(limit),
                                         None if bgu is None else _p(bgu), _p(gx)))
    return gx


def router_grad(x: np.ndarray, grad_out: np.ndarray, logits, idx: np.ndarray, renorm: bool, wgu: np.ndarray,
                wd: np.ndarray, tokens=None, act=ACT_SWIGLU, alpha=1.702, limit=7.0, bgu=None, bd=None):
    """fp64 gradient of L = <grad_out, y> with respect to the routing weights
    (dw [nt, k]) and, when logits are given, to the router logits (dlogits
    [nt, E]; else None), with the routing indices held."""
    x = np.ascontiguousarray(x, np.float64)
    g = np.ascontiguousarray(grad_out, np.float64)
    idx = np.ascontiguousarray(idx, np.int32)
    wgu = np.ascontiguousarray(wgu, np.float32)
    wd = np.ascontiguousarray(wd, np.float32)
    T, H = x.shape
    E, I2, _ = wgu.shape
    k = idx.shape[1]
    lg = None if logits is None else np.ascontiguousarray(logits, np.float32)
    El = E if lg is None else lg.shape[1]
    tok = None if tokens is None else np.ascontiguousarray(tokens, np.int64)
    nt = T if tok is None else tok.shape[0]
    dw = np.zeros((nt, k), np.float64)
    dl = None if lg is None else np.zeros((nt, El), np.float64)
    bgu, bd = _bias(bgu, (E, I2)), _bias(bd, (E, H))
    _check("e4bo_router_grad", _L().e4bo_router_grad(
        _p(x), _p(g), None if lg is None else _p(lg), T, El, H, I2 // 2, k, int(bool(renorm)), _p(idx), _p(wgu),
        _p(wd), None if tok is None else _p(tok), nt, int(act), float(alpha), float(limit),
        None if bgu is None else _p(bgu), None if bd is None else _p(bd), _p(dw), None if dl is None else _p(dl)))
    return dw, dl


def _lora(agu, bgu_l, ad, bd_l):
    agu, bgu_l, ad, bd_l = (np.ascontiguousarray(a, np.float32) for a in (agu, bgu_l, ad, bd_l))
    return agu, bgu_l, ad, bd_l, agu.shape[1]


def lora_forward(x, idx, w, wgu, wd, agu, bgu_l, ad, bd_l, scale, act=ACT_SWIGLU, alpha=1.702, limit=7.0, bgu=None,
                 bd=None) -> np.ndarray:
    """fp64 forward with per-expert LoRA adapters on both stacks: A_gu [E,r,H],
    B_gu [E,2I,r], A_d [E,r,I], B_d [E,H,r], update scale (alpha / r)."""
    x = np.ascontiguousarray(x, np.float64)
    idx = np.ascontiguousarray(idx, np.int32)
    w = np.ascontiguousarray(w, np.float64)
    wgu = np.ascontiguousarray(wgu, np.float32)
    wd = np.ascontiguousarray(wd, np.float32)
    agu, bgu_l, ad, bd_l, r = _lora(agu, bgu_l, ad, bd_l)
    T, H = x.shape
    E, I2, _ = wgu.shape
    k = idx.shape[1]
    y = np.zeros((T, H), np.float64)
    bgu, bd = _bias(bgu, (E, I2)), _bias(bd, (E, H))
    _check("e4bo_lora_forward", _L().e4bo_lora_forward(
        _p(x), T, E, H, I2 // 2, k, _p(idx), _p(w), _p(wgu), _p(wd), _p(agu), _p(bgu_l), _p(ad), _p(bd_l), r,
        float(scale), int(act), float(alpha), float(limit), None if bgu is None else _p(bgu),
        None if bd is None else _p(bd), _p(y)))
    return y


def lora_backward(x, grad_out, idx, w, wgu, wd, agu, bgu_l, ad, bd_l, scale, act=ACT_SWIGLU, alpha=1.702, limit=7.0,
                  bgu=None):
    """fp64 gradients of <grad_out, y> of lora_forward with the routing held and the
    base frozen: (grad_x [T,H], dA_gu, dB_gu, dA_d, dB_d) shaped like the adapters."""
    x = np.ascontiguousarray(x, np.float64)
    g = np.ascontiguousarray(grad_out, np.float64)
    idx = np.ascontiguousarray(idx, np.int32)
    w = np.ascontiguousarray(w, np.float64)
    wgu = np.ascontiguousarray(wgu, np.float32)
    wd = np.ascontiguousarray(wd, np.float32)
    agu, bgu_l, ad, bd_l, r = _lora(agu, bgu_l, ad, bd_l)
    T, H = x.shape
    E, I2, _ = wgu.shape
    k = idx.shape[1]
    gx = np.zeros((T, H), np.float64)
    out = [np.zeros(a.shape, np.float64) for a in (agu, bgu_l, ad, bd_l)]
    bgu = _bias(bgu, (E, I2))
    _check("e4bo_lora_backward", _L().e4bo_lora_backward(
        _p(x), _p(g), T, E, H, I2 // 2, k, _p(idx), _p(w), _p(wgu), _p(wd), _p(agu), _p(bgu_l), _p(ad), _p(bd_l), r,
        float(scale), int(act), float(alpha), float(limit), None if bgu is None else _p(bgu), _p(gx),
        *[_p(o) for o in out]))
    return (gx, *out)
