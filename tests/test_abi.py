"""CPU checks of the C-ABI library: it builds for sm_100a, loads, exports every
symbol include/e4b.h declares, and validates arguments on the host (no GPU
needed: every call here returns before any launch)."""
import ctypes
import os
import re

import pytest

from bit_quantized_mixture_nf4_b200 import build as e4b_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    e4b_build.build()
    import bit_quantized_mixture_nf4_b200 as e4b
    return e4b


def declared_functions():
    text = open(os.path.join(ROOT, "include", "e4b.h")).read()
    return sorted(set(re.findall(r"E4B_API\s+[\w\s\*]+?\b(e4b_\w+)\s*\(", text)))


def test_header_declares_the_four_operations():
    names = declared_functions()
    for n in ("e4b_quantize_nf4", "e4b_dequantize_nf4", "e4b_moe_forward", "e4b_moe_backward_dgrad"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    so = ctypes.CDLL(lib.LIB_PATH)
    for n in declared_functions():
        assert hasattr(so, n), n
    assert set(declared_functions()) == set(lib.EXPORTS)


def test_debug_build_exports_the_same_symbols_and_says_so(lib):
    """The debug-check build (E4B_DEBUG_CHECKS=1) has the same ABI; e4b_debug_checks
    (a host-only query) tells the two apart."""
    path = e4b_build.build(debug=True)
    dbg = ctypes.CDLL(path)
    for n in declared_functions():
        assert hasattr(dbg, n), n
    dbg.e4b_debug_checks.restype = ctypes.c_int
    rel = ctypes.CDLL(e4b_build.LIB)
    rel.e4b_debug_checks.restype = ctypes.c_int
    assert dbg.e4b_debug_checks() == 1
    assert rel.e4b_debug_checks() == 0


def test_status_strings(lib):
    for s in range(8):
        assert lib.e4b_status_string(s)
    assert lib.e4b_status_string(lib.E4B_ERR_DEBUG_CHECK) != lib.e4b_status_string(99)


def test_validate_schedule_rejects_bad_arguments_on_the_host(lib):
    L = lib.lib
    f = lambda P, E, tr, n: L.e4b_debug_validate_schedule(16, P, E, tr, 16, 16, 16, 16, n, 16, 16, None)
    assert f(0, 4, 256, 1) == lib.E4B_ERR_INVALID_ARG
    assert f(8, 0, 256, 1) == lib.E4B_ERR_INVALID_ARG
    assert f(8, 257, 256, 1) == lib.E4B_ERR_INVALID_ARG
    assert f(8, 4, 0, 1) == lib.E4B_ERR_INVALID_ARG
    assert f(8, 4, 256, -1) == lib.E4B_ERR_INVALID_ARG
    assert L.e4b_debug_validate_schedule(None, 8, 4, 256, 16, 16, 16, 16, 1, 16, 16, None) == lib.E4B_ERR_INVALID_ARG


def test_host_side_validation(lib):
    L = lib.lib
    nullp = None
    # quantize / dequantize: blocksize and in_features rules, null pointers
    assert L.e4b_quantize_nf4(nullp, 1, 2, 64, 32, 0, nullp, nullp, nullp) == lib.E4B_ERR_BLOCKSIZE
    assert L.e4b_quantize_nf4(nullp, 1, 2, 96, 64, 0, nullp, nullp, nullp) == lib.E4B_ERR_BLOCKSIZE
    assert L.e4b_quantize_nf4(nullp, 1, 2, 64, 64, 0, nullp, nullp, nullp) == lib.E4B_ERR_INVALID_ARG
    assert L.e4b_quantize_nf4(nullp, 1, 2, 64, 64, 5, nullp, nullp, nullp) == lib.E4B_ERR_INVALID_ARG
    assert L.e4b_quantize_nf4(nullp, 0, 2, 64, 64, 0, nullp, nullp, nullp) == lib.E4B_OK   # empty
    assert L.e4b_dequantize_nf4(nullp, nullp, 1, 2, 96, 64, 0, 1, nullp, nullp) == lib.E4B_ERR_BLOCKSIZE
    assert L.e4b_dequantize_nf4(nullp, nullp, 1, 2, 64, 64, 0, 7, nullp, nullp) == lib.E4B_ERR_INVALID_ARG
    # layer descriptions
    d = lib.make_desc(8, 256, 512, 2)
    assert lib.e4b_moe_workspace_size(d, 64) > 0
    for bad, code in ((lib.make_desc(8, 250, 512, 2), 0), (lib.make_desc(8, 256, 512, 9), 0),
                      (lib.make_desc(4, 256, 512, 5), 0), (lib.make_desc(300, 256, 512, 2), 0),
                      (lib.make_desc(8, 256, 512, 2, blocksize=128), 0)):
        assert lib.e4b_moe_workspace_size(bad, 64) == code
    ex = lib.e4b_experts(None, None, None, None)
    st = lambda: L.e4b_moe_forward(ctypes.byref(d), ctypes.byref(ex), None, 4, None, None, None, None, None,
                                   None, None, None, None, 0, None)
    assert st() == lib.E4B_ERR_INVALID_ARG
    ex2 = lib.e4b_experts(16, 16, 16, 16)   # non-null dummies: never dereferenced on these paths
    f = lambda dd, T, x, ws, n: L.e4b_moe_forward(ctypes.byref(dd), ctypes.byref(ex2), x, T, None, 16, 16, 16, None,
                                                  None, None, None, ws, n, None)
    assert f(d, 0, None, None, 0) == lib.E4B_OK                        # T == 0: no-op
    assert f(d, 4, None, 16, 1 << 30) == lib.E4B_ERR_INVALID_ARG       # null x
    assert f(d, 4, 16, None, 0) == lib.E4B_ERR_WORKSPACE               # no workspace
    assert f(d, 4, 16, 16, 10) == lib.E4B_ERR_WORKSPACE                # workspace too small
    bad_bs = lib.make_desc(8, 256, 512, 2, blocksize=32)
    assert f(bad_bs, 4, 16, 16, 1 << 30) == lib.E4B_ERR_BLOCKSIZE
    bad_h = lib.make_desc(8, 96, 512, 2)
    assert f(bad_h, 4, 16, 16, 1 << 30) == lib.E4B_ERR_BLOCKSIZE
    dec = lib.make_desc(8, 256, 512, 2, path=lib.PATH_DECODE)
    assert f(dec, 9, 16, 16, 1 << 40) == lib.E4B_ERR_UNSUPPORTED       # decode path is for T <= 8
    # activation: known kind, finite alpha, positive (possibly infinite) limit
    for bad in (lib.make_desc(8, 256, 512, 2, activation=2), lib.make_desc(8, 256, 512, 2, activation=-1),
                lib.make_desc(8, 256, 512, 2, activation=lib.ACT_CLAMPED_GLU, glu_limit=0.0),
                lib.make_desc(8, 256, 512, 2, activation=lib.ACT_CLAMPED_GLU, glu_limit=float("nan")),
                lib.make_desc(8, 256, 512, 2, activation=lib.ACT_CLAMPED_GLU, glu_alpha=float("inf"))):
        assert lib.e4b_moe_workspace_size(bad, 64) == 0
        assert f(bad, 4, 16, 16, 1 << 40) == lib.E4B_ERR_INVALID_ARG
    glu = lib.make_desc(8, 256, 512, 2, activation=lib.ACT_CLAMPED_GLU, glu_limit=float("inf"))
    assert lib.e4b_moe_workspace_size(glu, 64) == lib.e4b_moe_workspace_size(d, 64)
    # the decode kernels implement SwiGLU without biases: forcing them is refused before any launch
    glu_dec = lib.make_desc(8, 256, 512, 2, path=lib.PATH_DECODE, activation=lib.ACT_CLAMPED_GLU)
    assert f(glu_dec, 2, 16, 16, 1 << 40) == lib.E4B_ERR_UNSUPPORTED
    exb = lib.e4b_experts(16, 16, 16, 16, 16, None)
    assert L.e4b_moe_forward(ctypes.byref(dec), ctypes.byref(exb), 16, 2, None, 16, 16, 16, None, None, None, None,
                             16, 1 << 40, None) == lib.E4B_ERR_UNSUPPORTED
    # saved_h asks for the grouped path's intermediates: the decode path is refused
    assert L.e4b_moe_forward(ctypes.byref(dec), ctypes.byref(ex2), 16, 2, None, 16, 16, 16, None, 16, None, None,
                             16, 1 << 40, None) == lib.E4B_ERR_UNSUPPORTED
    g = lambda dd, T: L.e4b_moe_backward_dgrad(ctypes.byref(dd), ctypes.byref(ex2), None, T, 16, 16, 16, None, 16,
                                               16, 1 << 40, None)
    assert g(d, 4) == lib.E4B_ERR_INVALID_ARG                          # needs x when saved_gu is NULL
    assert g(d, 0) == lib.E4B_OK
    # the fused layer backward: argument rules, checked before any launch
    def b(T, x=16, logits=None, saved_gu=16, saved_h=16, gx=16, gw=16, gl=None):
        return L.e4b_moe_backward(ctypes.byref(d), ctypes.byref(ex2), x, T, logits, 16, 16, 16, saved_gu, saved_h,
                                  gx, gw, gl, None, None, 0, None)
    assert b(0) == lib.E4B_OK                                           # T == 0: no-op
    assert b(4, gx=None, gw=None) == lib.E4B_ERR_INVALID_ARG           # no output asked for
    assert b(4, x=None, saved_gu=None) == lib.E4B_ERR_INVALID_ARG      # nothing to recompute from
    assert b(4, saved_h=None) == lib.E4B_ERR_INVALID_ARG               # routing gradient needs the saved h
    assert b(4, gl=16) == lib.E4B_ERR_INVALID_ARG                      # grad_logits needs router_logits
    assert b(4, logits=16, gw=None, gl=16) == lib.E4B_ERR_INVALID_ARG  # ... and grad_topk_w
    assert b(4) == lib.E4B_ERR_WORKSPACE                               # valid request, no workspace
    # MXFP4: blocksize 32 with that codebook only; the scale arrays replace absmax
    mxd = lib.make_desc(8, 256, 512, 2, codebook=lib.MXFP4, blocksize=32)
    assert lib.e4b_moe_workspace_size(mxd, 64) > 0
    assert lib.e4b_moe_workspace_size(lib.make_desc(8, 256, 512, 2, codebook=lib.MXFP4), 64) == 0   # blocksize 64
    assert lib.e4b_moe_workspace_size(lib.make_desc(8, 256, 512, 2, blocksize=32), 64) == 0         # NF4 at 32
    assert f(mxd, 4, 16, 16, 1 << 40) == lib.E4B_ERR_INVALID_ARG      # scales missing
    assert lib.e4b_mxfp4_scale_stride(2880) == 96 and lib.e4b_mxfp4_scale_stride(512) == 16
    assert L.e4b_quantize_mxfp4(nullp, 1, 2, 48, nullp, nullp, nullp) == lib.E4B_ERR_BLOCKSIZE
    assert L.e4b_quantize_mxfp4(nullp, 1, 2, 64, nullp, nullp, nullp) == lib.E4B_ERR_INVALID_ARG
    assert L.e4b_dequantize_mxfp4(nullp, nullp, 1, 2, 64, 7, nullp, nullp) == lib.E4B_ERR_INVALID_ARG
    # 8-bit and bf16 storage: codebooks 3..5 at blocksize 64; anything past 5 is refused
    for cb in (lib.INT8, lib.FP8, lib.BF16_WEIGHTS):
        assert lib.e4b_moe_workspace_size(lib.make_desc(8, 256, 512, 2, codebook=cb), 64) > 0
    assert lib.e4b_moe_workspace_size(lib.make_desc(8, 256, 512, 2, codebook=6), 64) == 0
    # the 8-bit modes hold one stack dequantized to bf16 in the workspace
    assert (lib.e4b_moe_workspace_size(lib.make_desc(8, 256, 512, 2, codebook=lib.INT8), 64)
            >= lib.e4b_moe_workspace_size(d, 64) + 8 * 2 * 512 * 256 * 2)
    bfx = lib.e4b_experts(16, 16, None, None)   # bf16 passthrough needs no absmax
    bfd = lib.make_desc(8, 256, 512, 2, codebook=lib.BF16_WEIGHTS)
    assert L.e4b_moe_forward(ctypes.byref(bfd), ctypes.byref(bfx), 16, 4, None, 16, 16, 16, None, None, None, None,
                             16, 10, None) == lib.E4B_ERR_WORKSPACE
    assert L.e4b_quantize_nf4(nullp, 1, 2, 64, 64, lib.BF16_WEIGHTS, nullp, nullp, nullp) == lib.E4B_ERR_INVALID_ARG
    # LoRA: rank a multiple of 8 up to 64, finite scale, all four adapters present
    for bad in (lib.make_desc(8, 256, 512, 2, lora_rank=12), lib.make_desc(8, 256, 512, 2, lora_rank=72),
                lib.make_desc(8, 256, 512, 2, lora_rank=-8),
                lib.make_desc(8, 256, 512, 2, lora_rank=16, lora_scale=float("nan"))):
        assert lib.e4b_moe_workspace_size(bad, 64) == 0
    ld = lib.make_desc(8, 256, 512, 2, lora_rank=16, lora_scale=2.0)
    assert lib.e4b_moe_workspace_size(ld, 64) > lib.e4b_moe_workspace_size(d, 64)   # the thin operands
    assert f(ld, 4, 16, 16, 1 << 40) == lib.E4B_ERR_INVALID_ARG       # adapters missing
    exl = lib.e4b_experts(16, 16, 16, 16, None, None, 16, 16, 16, 16)
    ldec = lib.make_desc(8, 256, 512, 2, path=lib.PATH_DECODE, lora_rank=16, lora_scale=2.0)
    assert L.e4b_moe_forward(ctypes.byref(ldec), ctypes.byref(exl), 16, 2, None, 16, 16, 16, None, None, None, None,
                             16, 1 << 40, None) == lib.E4B_ERR_UNSUPPORTED   # decode kernels take no adapters
    gl = lib.e4b_lora_grads(16, 16, 16, 16)
    assert L.e4b_moe_backward(ctypes.byref(ld), ctypes.byref(exl), None, 4, None, 16, 16, 16, 16, 16, 16, None, None,
                              ctypes.byref(gl), None, 0, None) == lib.E4B_ERR_INVALID_ARG   # adapter grads need x


def test_pipe_host_side_validation(lib):
    """The pipelined runner rejects bad arguments before touching the device."""
    L = lib.lib
    d = lib.make_desc(8, 256, 512, 2)
    ex = lib.e4b_experts(16, 16, 16, 16)
    n = lib.e4b_pipe_arena_size(d, 64)
    assert n > lib.e4b_moe_workspace_size(d, 64)   # two input/output sets, saved g/u and the workspace
    assert lib.e4b_pipe_arena_size(lib.make_desc(8, 250, 512, 2), 64) == 0          # invalid desc
    out = ctypes.c_void_p()
    create = lambda dd, e, T, arena, nbytes: L.e4b_pipe_create(ctypes.byref(dd), ctypes.byref(e), T, arena, nbytes,
                                                               None, ctypes.byref(out))
    assert create(d, ex, 64, None, n) == lib.E4B_ERR_INVALID_ARG                    # no arena
    assert create(d, ex, 64, 256 + 16, n) == lib.E4B_ERR_INVALID_ARG                # arena not 256-byte aligned
    assert create(d, ex, -1, 256, n) == lib.E4B_ERR_INVALID_ARG                     # negative T_max
    assert create(d, ex, 64, 256, n - 1) == lib.E4B_ERR_WORKSPACE                   # arena too small
    assert create(d, lib.e4b_experts(None, 16, 16, 16), 64, 256, n) == lib.E4B_ERR_INVALID_ARG
    assert out.value is None
    assert L.e4b_pipe_submit(None, 4, 16, 16, 16, 16, 16) == lib.E4B_ERR_INVALID_ARG
    assert L.e4b_pipe_join(None) == lib.E4B_ERR_INVALID_ARG
    assert L.e4b_pipe_sync(None) == lib.E4B_ERR_INVALID_ARG
    L.e4b_pipe_destroy(None)   # a no-op
