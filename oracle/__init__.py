"""CPU oracle for the FP8-moment AdamW step -- TEST INFRASTRUCTURE.

Only the tests, the smoke check and the CPU-baseline leg of the benchmark may
import this package.  The library under ``fp8_quantized_adam_b200`` never
does, and the oracle never imports the library: the two share no code.

The arithmetic lives in ``fp8adam_oracle.c`` (plain scalar C, fp32 without
FMA contraction); this module compiles it with gcc and wraps it with ctypes.
Every function cites, in the C source, the page passage it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "fp8adam_oracle.c")
LIB = os.path.join(HERE, "liboracle_fp8adam.so")

# Format identifiers of the oracle.
E4M3, E5M2, FP32 = 0, 1, 2
FLAG_JIT_EVERY_STEP = 2

CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
          "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (idempotent); returns the library path."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, SRC, "-lm"])
        os.replace(tmp, LIB)
    return LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        L = _lib
        c_i64, c_u32, c_int, c_f = ctypes.c_int64, ctypes.c_uint32, ctypes.c_int, ctypes.c_float
        vp = ctypes.c_void_p
        L.ref_decode.restype = c_f
        L.ref_decode.argtypes = [c_int, c_u32]
        L.ref_fmax.restype = c_f
        L.ref_fmax.argtypes = [c_int]
        L.ref_encode.restype = c_u32
        L.ref_encode.argtypes = [c_int, c_f]
        L.ref_encode_array.restype = None
        L.ref_encode_array.argtypes = [c_int, vp, c_i64, vp]
        L.ref_encode_bits_range.restype = None
        L.ref_encode_bits_range.argtypes = [c_int, c_u32, c_i64, vp]
        L.ref_decode_array.restype = None
        L.ref_decode_array.argtypes = [c_int, vp, c_i64, vp]
        L.ref_pow2scale.restype = c_f
        L.ref_pow2scale.argtypes = [c_int, c_f, c_f, c_int]
        L.ref_step_constants.restype = None
        L.ref_step_constants.argtypes = [c_f, c_f, c_f, c_f, c_f, c_i64, vp]
        L.ref_fp8adam_step_tensor.restype = c_int
        L.ref_fp8adam_step_tensor.argtypes = [
            c_i64, vp, vp, vp, vp, vp, vp, vp, vp, c_int, c_int,
            c_f, c_f, c_f, c_f, c_f, c_i64, c_u32, vp]
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


# --------------------------------------------------------------------------
# codec
# --------------------------------------------------------------------------
def decode(fmt: int, codes) -> np.ndarray:
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, np.float32)
    lib().ref_decode_array(fmt, _ptr(c), c.size, _ptr(out))
    return out


def encode(fmt: int, x) -> np.ndarray:
    a = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(a.shape, np.uint8)
    lib().ref_encode_array(fmt, _ptr(a), a.size, _ptr(out))
    return out


def encode_bits_range(fmt: int, first: int, n: int) -> np.ndarray:
    """Codes of the floats whose bit patterns are first .. first+n-1."""
    out = np.empty(n, np.uint8)
    lib().ref_encode_bits_range(fmt, first, n, _ptr(out))
    return out


def fmax(fmt: int) -> float:
    return float(lib().ref_fmax(fmt))


def pow2scale(fmt: int, amax: float, s_prev: float, margin: int = 0) -> float:
    return float(lib().ref_pow2scale(fmt, amax, s_prev, margin))


def step_constants(lr, beta1, beta2, eps, wd, t) -> np.ndarray:
    out = np.empty(8, np.float32)
    lib().ref_step_constants(lr, beta1, beta2, eps, wd, t, _ptr(out))
    return out


# --------------------------------------------------------------------------
# the step
# --------------------------------------------------------------------------
class TensorState:
    """Host copy of one tensor's optimizer state (numpy, owned here)."""

    def __init__(self, p: np.ndarray, m_fmt: int, v_fmt: int,
                 m=None, v=None, scale_m=1.0, scale_v=1.0, amax_m=0.0, amax_v=0.0):
        self.p = np.ascontiguousarray(p, dtype=np.float32).copy()
        n = self.p.size
        self.m_fmt, self.v_fmt = m_fmt, v_fmt
        mdt = np.float32 if m_fmt == FP32 else np.uint8
        vdt = np.float32 if v_fmt == FP32 else np.uint8
        self.m = np.zeros(n, mdt) if m is None else np.ascontiguousarray(m, dtype=mdt).copy()
        self.v = np.zeros(n, vdt) if v is None else np.ascontiguousarray(v, dtype=vdt).copy()
        self.scale_m = np.array([scale_m], np.float32)
        self.scale_v = np.array([scale_v], np.float32)
        self.amax_m = np.array([amax_m], np.float32)
        self.amax_v = np.array([amax_v], np.float32)
        self.stats = np.zeros(2, np.uint64)

    def step(self, g_bits: np.ndarray, lr, beta1, beta2, eps, wd, t, flags=0):
        g = np.ascontiguousarray(g_bits, dtype=np.uint16)
        assert g.size == self.p.size
        rc = lib().ref_fp8adam_step_tensor(
            self.p.size, _ptr(self.p), _ptr(g), _ptr(self.m), _ptr(self.v),
            _ptr(self.scale_m), _ptr(self.scale_v), _ptr(self.amax_m), _ptr(self.amax_v),
            self.m_fmt, self.v_fmt, lr, beta1, beta2, eps, wd, t, flags, _ptr(self.stats))
        if rc != 0:
            raise ValueError("oracle step rejected its arguments (rc=%d)" % rc)
