"""e4b: NF4 / FP4 quantized Mixture-of-Experts expert kernels for NVIDIA B200.

A thin ctypes binding over ``libe4b.so`` (the C ABI in ``include/e4b.h``).  The
functions keep the C names and only marshal arguments: PyTorch tensors supply
device memory and the current CUDA stream; every step of the computation runs
in the library's sm_100a kernels.  There is no CPU fallback: the first call
fails loudly when the library is missing, and a compute call without a CUDA
device raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# E4B_DEBUG=1 loads the debug-check build (device-side bounds and schedule checks)
DEBUG = os.environ.get("E4B_DEBUG", "0") not in ("", "0")
LIB_PATH = os.path.join(_HERE, "libe4b_debug.so" if DEBUG else "libe4b.so")

E4B_OK, E4B_ERR_INVALID_ARG, E4B_ERR_BLOCKSIZE, E4B_ERR_UNSUPPORTED, E4B_ERR_WORKSPACE, E4B_ERR_CUDA, \
    E4B_ERR_TIMEOUT, E4B_ERR_DEBUG_CHECK = range(8)
# debug-check sites (bits 8..15 of e4b_last_status_word)
SITE_GEMM_TILE, SITE_GEMM_PERM, SITE_GATHER_PERM, SITE_COMBINE_INV, SITE_ROUTER_INV, SITE_OFFSETS, SITE_COUNTS, \
    SITE_TILE_PREFIX, SITE_SCHEDULE, SITE_PERM, SITE_INV_PERM = range(1, 12)
NF4, FP4, MXFP4, INT8, FP8, BF16_WEIGHTS = 0, 1, 2, 3, 4, 5   # storage formats (e4b_codebook)
F32, BF16 = 0, 1
PATH_AUTO, PATH_GROUPED, PATH_DECODE = 0, 1, 2
ACT_SWIGLU, ACT_CLAMPED_GLU = 0, 1

EXPORTS = ("e4b_quantize_nf4", "e4b_dequantize_nf4", "e4b_quantize_mxfp4", "e4b_dequantize_mxfp4",
           "e4b_mxfp4_scale_stride", "e4b_moe_workspace_size", "e4b_moe_forward",
           "e4b_moe_backward", "e4b_moe_backward_dgrad", "e4b_moe_backward_router", "e4b_device_status", "e4b_status_string",
           "e4b_launch_count", "e4b_timing_enable", "e4b_timing_enable_kinds", "e4b_timing_reset", "e4b_timing_get",
           "e4b_moe_forward_noalloc", "e4b_watchdog_selftest", "e4b_pipe_arena_size", "e4b_pipe_create",
           "e4b_pipe_submit", "e4b_pipe_join", "e4b_pipe_sync", "e4b_pipe_destroy", "e4b_last_status_word",
           "e4b_debug_checks", "e4b_debug_validate_schedule")
# kernel kinds of e4b_timing_get
KERNEL_KINDS = ("quantize", "dequantize", "route", "group", "gather", "combine", "gemm_gateup", "gemm_down",
                "gemm_dgrad_down", "gemm_dgrad_gateup", "decode_gateup", "decode_down")


class e4b_moe_desc(ctypes.Structure):
    _fields_ = [("E", ctypes.c_int), ("H", ctypes.c_int), ("I", ctypes.c_int), ("top_k", ctypes.c_int),
                ("renormalize", ctypes.c_int), ("codebook", ctypes.c_int), ("blocksize", ctypes.c_int),
                ("path", ctypes.c_int), ("activation", ctypes.c_int), ("glu_alpha", ctypes.c_float),
                ("glu_limit", ctypes.c_float), ("lora_rank", ctypes.c_int), ("lora_scale", ctypes.c_float)]


class e4b_experts(ctypes.Structure):
    _fields_ = [("gate_up", ctypes.c_void_p), ("down", ctypes.c_void_p), ("gate_up_absmax", ctypes.c_void_p),
                ("down_absmax", ctypes.c_void_p), ("gate_up_bias", ctypes.c_void_p), ("down_bias", ctypes.c_void_p),
                ("lora_A_gu", ctypes.c_void_p), ("lora_B_gu", ctypes.c_void_p), ("lora_A_d", ctypes.c_void_p),
                ("lora_B_d", ctypes.c_void_p), ("gate_up_scales", ctypes.c_void_p), ("down_scales", ctypes.c_void_p)]


class e4b_lora_grads(ctypes.Structure):
    _fields_ = [("dA_gu", ctypes.c_void_p), ("dB_gu", ctypes.c_void_p), ("dA_d", ctypes.c_void_p),
                ("dB_d", ctypes.c_void_p)]


class E4BError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: {msg} (status {status})")
        self.status = status


_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{os.path.basename(LIB_PATH)} not built at {LIB_PATH}; run "
                          f"python -m bit_quantized_mixture_nf4_b200.build --all")
    lib = ctypes.CDLL(LIB_PATH)
    P, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
    lib.e4b_quantize_nf4.argtypes = [P, i64, i64, i64, i32, i32, P, P, P]
    lib.e4b_dequantize_nf4.argtypes = [P, P, i64, i64, i64, i32, i32, i32, P, P]
    lib.e4b_quantize_mxfp4.argtypes = [P, i64, i64, i64, P, P, P]
    lib.e4b_dequantize_mxfp4.argtypes = [P, P, i64, i64, i64, i32, P, P]
    lib.e4b_mxfp4_scale_stride.argtypes = [i64]
    lib.e4b_mxfp4_scale_stride.restype = i64
    lib.e4b_moe_workspace_size.argtypes = [ctypes.POINTER(e4b_moe_desc), i64]
    lib.e4b_moe_workspace_size.restype = sz
    lib.e4b_moe_forward.argtypes = [ctypes.POINTER(e4b_moe_desc), ctypes.POINTER(e4b_experts), P, i64, P, P, P, P,
                                    P, P, P, P, P, sz, P]
    lib.e4b_moe_backward.argtypes = [ctypes.POINTER(e4b_moe_desc), ctypes.POINTER(e4b_experts), P, i64, P, P, P, P,
                                     P, P, P, P, P, P, P, sz, P]
    lib.e4b_moe_backward_dgrad.argtypes = [ctypes.POINTER(e4b_moe_desc), ctypes.POINTER(e4b_experts), P, i64, P, P,
                                           P, P, P, P, sz, P]
    lib.e4b_moe_forward_noalloc.argtypes = [ctypes.POINTER(e4b_moe_desc), ctypes.POINTER(e4b_experts), P, i64, P, P,
                                            P, P, P]
    lib.e4b_moe_backward_router.argtypes = [ctypes.POINTER(e4b_moe_desc), ctypes.POINTER(e4b_experts), P, i64, P, P,
                                            P, P, P, P, P, sz, P]
    lib.e4b_device_status.argtypes = [P]
    lib.e4b_last_status_word.argtypes = []
    lib.e4b_last_status_word.restype = ctypes.c_uint32
    lib.e4b_debug_checks.argtypes = []
    lib.e4b_debug_checks.restype = ctypes.c_int
    lib.e4b_debug_validate_schedule.argtypes = [P, i64, i32, i32, P, P, P, P, i64, P, P, P]
    lib.e4b_debug_validate_schedule.restype = ctypes.c_int
    lib.e4b_watchdog_selftest.argtypes = [P]
    lib.e4b_status_string.argtypes = [i32]
    lib.e4b_status_string.restype = ctypes.c_char_p
    lib.e4b_launch_count.restype = ctypes.c_uint64
    lib.e4b_timing_enable.argtypes = [i32]
    lib.e4b_timing_enable.restype = None
    lib.e4b_timing_enable_kinds.argtypes = [ctypes.c_uint32]
    lib.e4b_pipe_arena_size.argtypes = [ctypes.POINTER(e4b_moe_desc), i64]
    lib.e4b_pipe_arena_size.restype = sz
    lib.e4b_pipe_create.argtypes = [ctypes.POINTER(e4b_moe_desc), ctypes.POINTER(e4b_experts), i64, P, sz, P,
                                    ctypes.POINTER(ctypes.c_void_p)]
    lib.e4b_pipe_submit.argtypes = [P, i64, P, P, P, P, P]
    lib.e4b_pipe_join.argtypes = [P]
    lib.e4b_pipe_sync.argtypes = [P]
    lib.e4b_pipe_destroy.argtypes = [P]
    lib.e4b_pipe_destroy.restype = None
    lib.e4b_timing_enable_kinds.restype = None
    lib.e4b_timing_reset.restype = None
    lib.e4b_timing_get.argtypes = [i32, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_uint64)]
    lib.e4b_timing_get.restype = ctypes.c_int
    for f in ("e4b_quantize_nf4", "e4b_dequantize_nf4", "e4b_quantize_mxfp4", "e4b_dequantize_mxfp4",
              "e4b_moe_forward", "e4b_moe_backward", "e4b_moe_backward_dgrad",
              "e4b_device_status", "e4b_moe_forward_noalloc", "e4b_moe_backward_router", "e4b_watchdog_selftest"):
        getattr(lib, f).restype = ctypes.c_int
    _lib = lib
    return lib


def __getattr__(name):
    if name == "lib":
        return _load()
    raise AttributeError(name)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn: str, status: int):
    if status != E4B_OK:
        raise E4BError(fn, status, _load().e4b_status_string(status).decode())


def _cuda(t: torch.Tensor, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path)")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def e4b_status_string(status: int) -> str:
    return _load().e4b_status_string(status).decode()


def e4b_launch_count() -> int:
    return int(_load().e4b_launch_count())


def e4b_timing_enable(on: bool = True):
    _load().e4b_timing_enable(int(bool(on)))


def e4b_timing_enable_kinds(kinds):
    """Time only the given kernel kinds (indices or names in KERNEL_KINDS); empty turns timing off."""
    mask = 0
    for k in kinds:
        mask |= 1 << (KERNEL_KINDS.index(k) if isinstance(k, str) else int(k))
    _load().e4b_timing_enable_kinds(mask)


def e4b_timing_reset():
    _load().e4b_timing_reset()


def e4b_timing_get(kind) -> tuple:
    """(total device ms, timed launches) of one kernel kind (index or name in KERNEL_KINDS)."""
    if isinstance(kind, str):
        kind = KERNEL_KINDS.index(kind)
    ms, n = ctypes.c_double(), ctypes.c_uint64()
    _check("e4b_timing_get", _load().e4b_timing_get(kind, ctypes.byref(ms), ctypes.byref(n)))
    return ms.value, int(n.value)


def e4b_device_status(stream=None) -> int:
    return int(_load().e4b_device_status(_stream(stream)))


def e4b_last_status_word() -> int:
    """Raw status word of the last e4b_device_status call (bits 8..15: debug-check site)."""
    return int(_load().e4b_last_status_word())


def e4b_debug_checks() -> bool:
    """True when the loaded library is the debug-check build."""
    return bool(_load().e4b_debug_checks())


def e4b_debug_validate_schedule(topk_idx, E: int, tile_rows: int, counts, offsets, tile_prefix, sched, perm, inv_perm,
                                stream=None) -> int:
    """Checks a grouping schedule on the device; returns the status (E4B_OK or
    E4B_ERR_DEBUG_CHECK, the failing site then in e4b_last_status_word() >> 8)."""
    for t, n in ((topk_idx, "topk_idx"), (counts, "counts"), (offsets, "offsets"), (tile_prefix, "tile_prefix"),
                 (sched, "sched"), (perm, "perm"), (inv_perm, "inv_perm")):
        _cuda(t, n, torch.int32)
    if sched.dim() != 2 or sched.shape[1] != 4:
        raise ValueError("sched must be [n, 4] int32")
    return int(_load().e4b_debug_validate_schedule(_ptr(topk_idx), topk_idx.numel(), E, tile_rows, _ptr(counts),
                                                   _ptr(offsets), _ptr(tile_prefix), _ptr(sched), sched.shape[0],
                                                   _ptr(perm), _ptr(inv_perm), _stream(stream)))


def e4b_quantize_nf4(w: torch.Tensor, blocksize: int = 64, codebook: int = NF4, packed=None, absmax=None,
                     stream=None):
    """w: fp32 [E, out, in] on the GPU -> (packed uint8 [E, out*in/2] (the 8-bit
    codebooks INT8 / FP8: [E, out*in], one byte per element), absmax fp32 [E, out*in/64])."""
    _cuda(w, "w", torch.float32)
    if w.dim() != 3:
        raise ValueError("w must be a 3-D [E, out, in] stack")
    E, o, i = w.shape
    if packed is None:
        packed = torch.empty(E, o * i // (1 if codebook in (INT8, FP8) else 2), dtype=torch.uint8, device=w.device)
    if absmax is None:
        absmax = torch.empty(E, o * i // max(blocksize, 1), dtype=torch.float32, device=w.device)
    _check("e4b_quantize_nf4", _load().e4b_quantize_nf4(_ptr(w), E, o, i, blocksize, codebook, _ptr(packed), _ptr(absmax),
                                                    _stream(stream)))
    return packed, absmax


def e4b_dequantize_nf4(packed: torch.Tensor, absmax: torch.Tensor, shape, blocksize: int = 64, codebook: int = NF4,
                       out_dtype: int = BF16, out=None, stream=None):
    """Packed + absmax -> [E, out, in] bf16 (out_dtype=BF16) or fp32 (F32)."""
    _cuda(packed, "packed", torch.uint8)
    _cuda(absmax, "absmax", torch.float32)
    E, o, i = shape
    if out is None:
        out = torch.empty(E, o, i, dtype=torch.bfloat16 if out_dtype == BF16 else torch.float32, device=packed.device)
    _check("e4b_dequantize_nf4", _load().e4b_dequantize_nf4(_ptr(packed), _ptr(absmax), E, o, i, blocksize, codebook,
                                                        out_dtype, _ptr(out), _stream(stream)))
    return out


def make_desc(E, H, I, top_k, renormalize=True, codebook=NF4, blocksize=64, path=PATH_AUTO, activation=ACT_SWIGLU,
              glu_alpha=1.702, glu_limit=7.0, lora_rank=0, lora_scale=1.0) -> e4b_moe_desc:
    return e4b_moe_desc(E, H, I, top_k, int(bool(renormalize)), codebook, blocksize, path, activation, glu_alpha,
                        glu_limit, lora_rank, lora_scale)


def e4b_mxfp4_scale_stride(cols: int) -> int:
    return int(_load().e4b_mxfp4_scale_stride(cols))


def e4b_quantize_mxfp4(w: torch.Tensor, stream=None):
    """fp32 [E, out, in] (CUDA) -> (packed uint8 [E, out*in/2], scales uint8 [E, out, S]):
    OCP MX v1.0 MXFP4 (32-element blocks, E8M0 scales, E2M1 codes)."""
    _cuda(w, "w", torch.float32)
    if w.dim() != 3 or not w.is_contiguous():
        raise ValueError("w must be a contiguous [E, out, in] tensor")
    E, o, i = w.shape
    packed = torch.empty(E, o * i // 2, dtype=torch.uint8, device=w.device)
    scales = torch.empty(E, o, e4b_mxfp4_scale_stride(i), dtype=torch.uint8, device=w.device)
    _check("e4b_quantize_mxfp4", _load().e4b_quantize_mxfp4(_ptr(w), E, o, i, _ptr(packed), _ptr(scales),
                                                          _stream(stream)))
    return packed, scales


def e4b_dequantize_mxfp4(packed: torch.Tensor, scales: torch.Tensor, shape, out_dtype=torch.bfloat16, stream=None):
    _cuda(packed, "packed", torch.uint8)
    _cuda(scales, "scales", torch.uint8)
    E, o, i = shape
    out = torch.empty(E, o, i, dtype=out_dtype, device=packed.device)
    _check("e4b_dequantize_mxfp4", _load().e4b_dequantize_mxfp4(
        _ptr(packed), _ptr(scales), E, o, i, BF16 if out_dtype == torch.bfloat16 else F32, _ptr(out),
        _stream(stream)))
    return out


def make_experts(gate_up, down, gate_up_absmax, down_absmax, gate_up_bias=None, down_bias=None,
                 lora=None, gate_up_scales=None, down_scales=None) -> e4b_experts:
    """The two packed stacks and their absmax (device tensors), plus optional fp32
    per-expert biases gate_up_bias [E, 2I] and down_bias [E, H], and optional bf16
    LoRA adapters lora = (A_gu [E, r, H], B_gu [E, 2I, r], A_d [E, r, I], B_d [E, H, r])
    (the descriptor's lora_rank must be r).  The tensors must outlive every call
    that uses the returned struct."""
    for n, t in (("gate_up", gate_up), ("down", down)):
        _cuda(t, n, torch.uint8)
    for n, t in (("gate_up_absmax", gate_up_absmax), ("down_absmax", down_absmax)):
        if t is not None:
            _cuda(t, n, torch.float32)
    for n, t in (("gate_up_scales", gate_up_scales), ("down_scales", down_scales)):
        if t is not None:
            _cuda(t, n, torch.uint8)
    for n, t in (("gate_up_bias", gate_up_bias), ("down_bias", down_bias)):
        if t is not None:
            _cuda(t, n, torch.float32)
    ad = [None] * 4
    if lora is not None:
        for i, (n, t) in enumerate(zip(("A_gu", "B_gu", "A_d", "B_d"), lora)):
            _cuda(t, n, torch.bfloat16)
            if not t.is_contiguous():
                raise ValueError(f"{n} must be contiguous")
            ad[i] = t.data_ptr()
    ptr = lambda t: None if t is None else t.data_ptr()
    return e4b_experts(gate_up.data_ptr(), down.data_ptr(), ptr(gate_up_absmax), ptr(down_absmax),
                       ptr(gate_up_bias), ptr(down_bias), *ad, ptr(gate_up_scales), ptr(down_scales))


def e4b_moe_workspace_size(desc: e4b_moe_desc, T: int) -> int:
    return int(_load().e4b_moe_workspace_size(ctypes.byref(desc), T))


def workspace(desc: e4b_moe_desc, T: int, device="cuda") -> torch.Tensor:
    return torch.empty(max(e4b_moe_workspace_size(desc, T), 1), dtype=torch.uint8, device=device)


def e4b_moe_forward(desc: e4b_moe_desc, experts: e4b_experts, x: torch.Tensor, router_logits=None, topk_idx=None,
                    topk_w=None, y=None, saved_gu=None, offsets_out=None, perm_out=None, ws=None, stream=None,
                    saved_h=None):
    """Expert-layer forward.  With router_logits the layer routes and fills
    topk_idx / topk_w (allocated here when not given); without, they are inputs.
    Returns (y, topk_idx, topk_w)."""
    _cuda(x, "x", torch.bfloat16)
    T = x.shape[0]
    dev = x.device
    if topk_idx is None:
        topk_idx = torch.empty(T, desc.top_k, dtype=torch.int32, device=dev)
    if topk_w is None:
        topk_w = torch.empty(T, desc.top_k, dtype=torch.float32, device=dev)
    if router_logits is not None:
        _cuda(router_logits, "router_logits", torch.float32)
    if y is None:
        y = torch.empty(T, desc.H, dtype=torch.bfloat16, device=dev)
    if ws is None:
        ws = workspace(desc, T, dev)
    _check("e4b_moe_forward", _load().e4b_moe_forward(
        ctypes.byref(desc), ctypes.byref(experts), _ptr(x), T, _ptr(router_logits), _ptr(topk_idx), _ptr(topk_w),
        _ptr(y), _ptr(saved_gu), _ptr(saved_h), _ptr(offsets_out), _ptr(perm_out), _ptr(ws), ws.numel(),
        _stream(stream)))
    return y, topk_idx, topk_w


def e4b_moe_backward(desc: e4b_moe_desc, experts: e4b_experts, x, topk_idx, topk_w, grad_out, saved_gu=None,
                     saved_h=None, router_logits=None, grad_x=None, grad_topk_w=None, grad_logits=None,
                     want_grad_x=True, want_routing=True, lora_grads=None, ws=None, stream=None):
    """The layer backward in one pass: (grad_x bf16 [T, H] or None, grad_topk_w fp32
    [T, k] or None, grad_logits fp32 [T, E] or None).  The routing-weight gradient
    is fused into the input gradient's down^T GEMM; with saved_gu it needs
    saved_h (both from e4b_moe_forward), without them x is used to recompute.
    lora_grads: fp32 tensors (dA_gu, dB_gu, dA_d, dB_d) shaped like the adapters,
    written with the adapter gradients (needs x)."""
    _cuda(grad_out, "grad_out", torch.bfloat16)
    T = grad_out.shape[0]
    dev = grad_out.device
    if grad_x is None and want_grad_x:
        grad_x = torch.empty(T, desc.H, dtype=torch.bfloat16, device=dev)
    if grad_topk_w is None and want_routing:
        grad_topk_w = torch.empty(T, desc.top_k, dtype=torch.float32, device=dev)
    if router_logits is not None:
        _cuda(router_logits, "router_logits", torch.float32)
        if grad_logits is None and want_routing:
            grad_logits = torch.empty(T, desc.E, dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace(desc, T, dev)
    lg = None
    if lora_grads is not None:
        for n, t in zip(("dA_gu", "dB_gu", "dA_d", "dB_d"), lora_grads):
            _cuda(t, n, torch.float32)
        lg = e4b_lora_grads(*[t.data_ptr() for t in lora_grads])
    _check("e4b_moe_backward", _load().e4b_moe_backward(
        ctypes.byref(desc), ctypes.byref(experts), _ptr(x), T, _ptr(router_logits), _ptr(topk_idx), _ptr(topk_w),
        _ptr(grad_out), _ptr(saved_gu), _ptr(saved_h), _ptr(grad_x), _ptr(grad_topk_w), _ptr(grad_logits),
        None if lg is None else ctypes.byref(lg), _ptr(ws), ws.numel(), _stream(stream)))
    return grad_x, grad_topk_w, grad_logits


def e4b_moe_backward_dgrad(desc: e4b_moe_desc, experts: e4b_experts, x, topk_idx, topk_w, grad_out, saved_gu=None,
                           grad_x=None, ws=None, stream=None):
    """Input gradient with routing held constant; returns grad_x bf16 [T, H]."""
    _cuda(grad_out, "grad_out", torch.bfloat16)
    T = grad_out.shape[0]
    dev = grad_out.device
    if grad_x is None:
        grad_x = torch.empty(T, desc.H, dtype=torch.bfloat16, device=dev)
    if ws is None:
        ws = workspace(desc, T, dev)
    _check("e4b_moe_backward_dgrad", _load().e4b_moe_backward_dgrad(
        ctypes.byref(desc), ctypes.byref(experts), _ptr(x), T, _ptr(topk_idx), _ptr(topk_w), _ptr(grad_out),
        _ptr(saved_gu), _ptr(grad_x), _ptr(ws), ws.numel(), _stream(stream)))
    return grad_x


def e4b_moe_forward_noalloc(desc: e4b_moe_desc, experts: e4b_experts, x: torch.Tensor, router_logits=None,
                            topk_idx=None, topk_w=None, y=None, stream=None):
    """The forward with the library's own fixed scratch (no workspace argument).
    Output tensors are allocated here only when not given.  Returns (y, topk_idx, topk_w)."""
    _cuda(x, "x", torch.bfloat16)
    T = x.shape[0]
    dev = x.device
    if topk_idx is None:
        topk_idx = torch.empty(T, desc.top_k, dtype=torch.int32, device=dev)
    if topk_w is None:
        topk_w = torch.empty(T, desc.top_k, dtype=torch.float32, device=dev)
    if router_logits is not None:
        _cuda(router_logits, "router_logits", torch.float32)
    if y is None:
        y = torch.empty(T, desc.H, dtype=torch.bfloat16, device=dev)
    _check("e4b_moe_forward_noalloc", _load().e4b_moe_forward_noalloc(
        ctypes.byref(desc), ctypes.byref(experts), _ptr(x), T, _ptr(router_logits), _ptr(topk_idx), _ptr(topk_w),
        _ptr(y), _stream(stream)))
    return y, topk_idx, topk_w


def e4b_moe_backward_router(desc: e4b_moe_desc, experts: e4b_experts, x, topk_idx, topk_w, grad_out,
                            router_logits=None, grad_topk_w=None, grad_logits=None, want_logits=True, ws=None,
                            stream=None):
    """Routing gradient with the indices held: (grad_topk_w fp32 [T, k],
    grad_logits fp32 [T, E] or None).  grad_logits needs router_logits."""
    _cuda(x, "x", torch.bfloat16)
    _cuda(grad_out, "grad_out", torch.bfloat16)
    T = x.shape[0]
    dev = x.device
    if grad_topk_w is None:
        grad_topk_w = torch.empty(T, desc.top_k, dtype=torch.float32, device=dev)
    if router_logits is not None:
        _cuda(router_logits, "router_logits", torch.float32)
        if grad_logits is None and want_logits:
            grad_logits = torch.empty(T, desc.E, dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace(desc, T, dev)
    _check("e4b_moe_backward_router", _load().e4b_moe_backward_router(
        ctypes.byref(desc), ctypes.byref(experts), _ptr(x), T, _ptr(router_logits), _ptr(topk_idx), _ptr(topk_w),
        _ptr(grad_out), _ptr(grad_topk_w), _ptr(grad_logits), _ptr(ws), ws.numel(), _stream(stream)))
    return grad_topk_w, grad_logits


def e4b_watchdog_selftest(stream=None):
    """Launch the watchdog self-test kernel (a bounded wait that must time out)."""
    _check("e4b_watchdog_selftest", _load().e4b_watchdog_selftest(_stream(stream)))


# ------------------------------------------------------------- pipelined host-buffer steps

def _host(t: torch.Tensor, name: str, dtype, shape):
    if t.is_cuda or not t.is_pinned():
        raise ValueError(f"{name} must be a page-locked host tensor (pin_memory())")
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)}")
    return ctypes.c_void_p(t.data_ptr())


def e4b_pipe_arena_size(desc: e4b_moe_desc, T_max: int) -> int:
    return int(_load().e4b_pipe_arena_size(ctypes.byref(desc), T_max))


class e4b_pipe:
    """Handle of a pipelined host-buffer step runner (e4b_pipe_create): owns the
    device arena tensor and keeps the descriptor and expert tensors alive."""

    def __init__(self, handle, arena, desc, experts, T_max):
        self.handle, self.arena, self.desc, self.experts, self.T_max = handle, arena, desc, experts, T_max


def e4b_pipe_create(desc: e4b_moe_desc, experts: e4b_experts, T_max: int, device="cuda", stream=None) -> e4b_pipe:
    size = e4b_pipe_arena_size(desc, T_max)
    if size == 0:
        raise ValueError("invalid descriptor or T_max")
    arena = torch.empty(size, dtype=torch.uint8, device=device)
    h = ctypes.c_void_p()
    _check("e4b_pipe_create", _load().e4b_pipe_create(ctypes.byref(desc), ctypes.byref(experts), T_max,
                                                      _ptr(arena), size, _stream(stream), ctypes.byref(h)))
    return e4b_pipe(h, arena, desc, experts, T_max)


def e4b_pipe_submit(pipe: e4b_pipe, x, router_logits, grad_out, y, grad_x):
    """Enqueue one batch: pinned host x [T,H] bf16, router_logits [T,E] fp32,
    grad_out [T,H] bf16 in; pinned host y and grad_x [T,H] bf16 out (valid after
    a later e4b_pipe_join/e4b_pipe_sync)."""
    d = pipe.desc
    T = x.shape[0]
    args = (_host(x, "x", torch.bfloat16, (T, d.H)), _host(router_logits, "router_logits", torch.float32, (T, d.E)),
            _host(grad_out, "grad_out", torch.bfloat16, (T, d.H)), _host(y, "y", torch.bfloat16, (T, d.H)),
            _host(grad_x, "grad_x", torch.bfloat16, (T, d.H)))
    _check("e4b_pipe_submit", _load().e4b_pipe_submit(pipe.handle, T, *args))


def e4b_pipe_join(pipe: e4b_pipe):
    _check("e4b_pipe_join", _load().e4b_pipe_join(pipe.handle))


def e4b_pipe_sync(pipe: e4b_pipe):
    _check("e4b_pipe_sync", _load().e4b_pipe_sync(pipe.handle))


def e4b_pipe_destroy(pipe: e4b_pipe):
    if pipe.handle:
        _load().e4b_pipe_destroy(pipe.handle)
        pipe.handle = None
