"""Builds libe4b.so (the CUDA kernels and the C ABI) in-tree for sm_100a, and
libe4b_debug.so, the same sources with the device-side bounds and schedule checks
compiled in (E4B_DEBUG_CHECKS=1; the package loads it when E4B_DEBUG=1).

    python -m bit_quantized_mixture_nf4_b200.build [--force] [--debug | --all]

nvcc cross-compiles without a GPU.  The CUDA runtime is linked statically so the
library does not depend on which libcudart the host process loaded first.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libe4b.so")
DEBUG_LIB = os.path.join(PKG, "libe4b_debug.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Builds the release library (debug=False) or the debug-check one; returns its path."""
    lib = DEBUG_LIB if debug else LIB
    if not force and not _stale(lib):
        return lib
    objdir = os.path.join(ROOT, "_build_debug" if debug else "_build")
    os.makedirs(objdir, exist_ok=True)
    defs = ["-DE4B_DEBUG_CHECKS=1"] if debug else []
    objs = []
    procs = []
    for src in sources():
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [NVCC, *ARCH, *FLAGS, *defs, "-c", src, "-o", obj]
        if verbose:
            cmd += ["-Xptxas", "-v"]
        procs.append((cmd, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)))
        objs.append(obj)
    failed = False
    for cmd, pr in procs:
        out, _ = pr.communicate()
        if out and (verbose or pr.returncode):
            sys.stderr.write(out)
        if pr.returncode:
            failed = True
            sys.stderr.write("FAILED: " + " ".join(cmd) + "\n")
    if failed:
        raise RuntimeError("nvcc failed")
    tmp = lib + f".tmp{os.getpid()}"
    subprocess.run([NVCC, *ARCH, "-shared", "-o", tmp, *objs, "-cudart", "static"], check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    force, verbose = "--force" in sys.argv, "-v" in sys.argv
    if "--all" in sys.argv or "--debug" not in sys.argv:
        print(build(force=force, verbose=verbose))
    if "--all" in sys.argv or "--debug" in sys.argv:
        print(build(force=force, verbose=verbose, debug=True))
