"""Build ``libfp8adam.so`` in-tree with nvcc for sm_100a.

The library is plain CUDA C++ with a C ABI (include/fp8adam.h); it links
only the CUDA runtime (static), not torch.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libfp8adam.so")
LIB_DEBUG = os.path.join(PKG, "libfp8adam_debug.so")  # bounds checks, wait injection (FP8ADAM_DEBUG)
SOURCES = [os.path.join(CSRC, "fp8adam_capi.cu"), os.path.join(CSRC, "fp8adam_noalloc.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("fp8_codec.cuh", "fp8adam_step.cuh", "fp8adam_ext.cuh", "fp8adam_step_tma.cuh", "fp8adam_ext_tma.cuh", "fp8adam_debug.cuh")] + [
    os.path.join(ROOT, "include", "fp8adam.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-fmad=false",  # every fp32 operation of the step is a single rounding
    "-Xcompiler", "-fPIC", "-shared",
    "-I", os.path.join(ROOT, "include"),
]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.sep not in c or os.path.exists(c)):
            return c
    raise RuntimeError("nvcc not found")


def _build_one(lib: str, flags, force: bool, verbose: bool) -> str:
    newest = max(os.path.getmtime(p) for p in DEPS)
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= newest:
        return lib
    tmp = lib + ".tmp%d" % os.getpid()
    cmd = [nvcc(), *NVCC_FLAGS, *flags, "-o", tmp, *SOURCES]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


def build(force: bool = False, verbose: bool = False, extra=(), debug: bool = True) -> str:
    """The release library (returned) and, unless debug=False, the debug one."""
    if extra:
        force = True
    lib = _build_one(LIB, list(extra), force, verbose)
    if debug:
        _build_one(LIB_DEBUG, ["-DFP8ADAM_DEBUG", *extra], force, verbose)
    return lib


if __name__ == "__main__":
    build(force=True, verbose=True, extra=sys.argv[1:])
