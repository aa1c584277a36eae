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
FLAG_UPDATE_FROM_STORED = 4
FLAG_STOCHASTIC = 8
FLAG_SR_DRAW16 = 32  # with FLAG_STOCHASTIC: 16-bit draws


class StepOpts(ctypes.Structure):
    """Options of the extended step (mirrors ref_step_opts in the C source)."""
    _fields_ = [("flags", ctypes.c_uint32), ("margin_m", ctypes.c_int32), ("margin_v", ctypes.c_int32),
                ("hist_len", ctypes.c_int32), ("hist_m", ctypes.c_void_p), ("hist_v", ctypes.c_void_p),
                ("seed", ctypes.c_uint64), ("tensor_index", ctypes.c_int32), ("grad_mult", ctypes.c_float),
                ("skip", ctypes.c_int32), ("p_bf16", ctypes.c_void_p)]

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
        L.ref_fp8adam_step_tensor_ex.restype = c_int
        L.ref_fp8adam_step_tensor_ex.argtypes = [
            c_i64, vp, vp, vp, vp, vp, vp, vp, vp, c_int, c_int,
            c_f, c_f, c_f, c_f, c_f, c_i64, c_u32, ctypes.POINTER(StepOpts), vp]
        L.ref_philox4x32_10.restype = None
        L.ref_philox4x32_10.argtypes = [vp, vp, vp]
        L.ref_sr_bits.restype = c_u32
        L.ref_sr_bits.argtypes = [ctypes.c_uint64, ctypes.c_int32, c_i64, c_i64, c_int]
        L.ref_encode_sr.restype = c_u32
        L.ref_encode_sr.argtypes = [c_int, c_f, c_u32]
        L.ref_encode_sr_array.restype = None
        L.ref_encode_sr_array.argtypes = [c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, c_i64]
        L.ref_rev16.restype = c_u32
        L.ref_rev16.argtypes = [c_u32]
        L.ref_sr16_draw.restype = c_u32
        L.ref_sr16_draw.argtypes = [c_u32, c_int]
        L.ref_encode_sr16.restype = c_u32
        L.ref_encode_sr16.argtypes = [c_int, c_f, c_u32]
        L.ref_encode_sr16_array.restype = None
        L.ref_encode_sr16_array.argtypes = [c_int, vp, vp, vp, c_i64]
        L.ref_encode_sr16_words.restype = None
        L.ref_encode_sr16_words.argtypes = [c_int, vp, vp, vp, c_i64]
        L.ref_sr16_bits.restype = c_u32
        L.ref_sr16_bits.argtypes = [ctypes.c_uint64, ctypes.c_int32, c_i64, c_i64, c_int]
        L.ref_f32_to_bf16.restype = ctypes.c_uint16
        L.ref_f32_to_bf16.argtypes = [c_f]
        L.ref_f32_to_bf16_array.restype = None
        L.ref_f32_to_bf16_array.argtypes = [vp, c_i64, vp]
        L.ref_grad_sumsq.restype = None
        L.ref_grad_sumsq.argtypes = [ctypes.c_int32, vp, vp, vp, vp]
        L.ref_grad_multiplier.restype = c_f
        L.ref_grad_multiplier.argtypes = [ctypes.c_double, c_f, c_f]
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


def philox4x32_10(ctr, key) -> list:
    c = np.asarray(ctr, np.uint32)
    k = np.asarray(key, np.uint32)
    out = np.empty(4, np.uint32)
    lib().ref_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return [int(x) for x in out]


def sr_bits(seed: int, tensor: int, t: int, j: int, which: int) -> int:
    return int(lib().ref_sr_bits(seed, tensor, t, j, which))


def encode_sr(fmt: int, x: float, r: int) -> int:
    return int(lib().ref_encode_sr(fmt, x, r))


def rev16(x: int) -> int:
    return int(lib().ref_rev16(x))


def sr16_draw(w: int, k: int) -> int:
    """The 16-bit draw of code k (0..3) among the four codes word w serves."""
    return int(lib().ref_sr16_draw(w, k))


def encode_sr16(fmt: int, x: float, r16: int) -> int:
    return int(lib().ref_encode_sr16(fmt, x, r16))


def encode_sr16_array(fmt: int, x, r16) -> np.ndarray:
    """Codes of x[j] stochastically rounded with the 16-bit draws r16[j]."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    r = np.ascontiguousarray(r16, dtype=np.uint32)
    assert x.shape == r.shape
    out = np.empty(x.size, np.uint8)
    lib().ref_encode_sr16_array(fmt, _ptr(x), _ptr(r), _ptr(out), x.size)
    return out


def encode_sr16_words(fmt: int, x, w) -> np.ndarray:
    """Codes of x[j] with the draw of code j % 4 of word w[j // 4]."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    w = np.ascontiguousarray(w, dtype=np.uint32)
    assert w.size * 4 >= x.size
    out = np.empty(x.size, np.uint8)
    lib().ref_encode_sr16_words(fmt, _ptr(x), _ptr(w), _ptr(out), x.size)
    return out


def sr16_bits(seed: int, tensor: int, t: int, j: int, which: int) -> int:
    return int(lib().ref_sr16_bits(seed, tensor, t, j, which))


def encode_sr_array(fmt: int, x, r) -> np.ndarray:
    """Codes of x[j] stochastically rounded with the random words r[j]."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    r = np.ascontiguousarray(r, dtype=np.uint32)
    assert x.shape == r.shape
    out = np.empty(x.size, np.uint8)
    lib().ref_encode_sr_array(fmt, _ptr(x), _ptr(r), _ptr(out), x.size)
    return out


def f32_to_bf16(x) -> np.ndarray:
    a = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(a.shape, np.uint16)
    lib().ref_f32_to_bf16_array(_ptr(a), a.size, _ptr(out))
    return out


def grad_sumsq(grads) -> tuple:
    """(exact sum of g^2 rounded to double, non-finite count) over a list of
    bf16-bit numpy arrays."""
    arrs = [np.ascontiguousarray(g, dtype=np.uint16) for g in grads]
    n = np.array([a.size for a in arrs], np.int64)
    ptrs = np.array([a.ctypes.data for a in arrs], np.uint64)
    s = ctypes.c_double()
    bad = ctypes.c_uint64()
    lib().ref_grad_sumsq(len(arrs), _ptr(n), _ptr(ptrs), ctypes.addressof(s), ctypes.addressof(bad))
    return s.value, bad.value


def grad_multiplier(sumsq: float, loss_scale: float, max_norm: float) -> float:
    return float(lib().ref_grad_multiplier(sumsq, loss_scale, max_norm))


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

    def step_ex(self, g_bits: np.ndarray, lr, beta1, beta2, eps, wd, t, flags=0, *, margin_m=0,
                margin_v=0, hist_len=0, seed=0, tensor_index=0, grad_mult=1.0, skip=False,
                want_bf16=False):
        """The extended step (scaling/read-back variants, stochastic rounding,
        gradient multiplier, bf16 param copy); state kept on this object."""
        g = np.ascontiguousarray(g_bits, dtype=np.uint16)
        assert g.size == self.p.size
        if hist_len > 1 and getattr(self, "hist_m", None) is None:
            self.hist_m = np.zeros(hist_len, np.float32)
            self.hist_v = np.zeros(hist_len, np.float32)
        self.p_bf16 = np.zeros(self.p.size, np.uint16) if want_bf16 else None
        o = StepOpts(flags, margin_m, margin_v, hist_len,
                     _ptr(self.hist_m) if hist_len > 1 else None,
                     _ptr(self.hist_v) if hist_len > 1 else None,
                     seed, tensor_index, grad_mult, 1 if skip else 0,
                     _ptr(self.p_bf16) if want_bf16 else None)
        rc = lib().ref_fp8adam_step_tensor_ex(
            self.p.size, _ptr(self.p), _ptr(g), _ptr(self.m), _ptr(self.v),
            _ptr(self.scale_m), _ptr(self.scale_v), _ptr(self.amax_m), _ptr(self.amax_v),
            self.m_fmt, self.v_fmt, lr, beta1, beta2, eps, wd, t, flags, ctypes.byref(o),
            _ptr(self.stats))
        if rc != 0:
            raise ValueError("oracle step rejected its arguments (rc=%d)" % rc)

    def step(self, g_bits: np.ndarray, lr, beta1, beta2, eps, wd, t, flags=0):
        g = np.ascontiguousarray(g_bits, dtype=np.uint16)
        assert g.size == self.p.size
        rc = lib().ref_fp8adam_step_tensor(
            self.p.size, _ptr(self.p), _ptr(g), _ptr(self.m), _ptr(self.v),
            _ptr(self.scale_m), _ptr(self.scale_v), _ptr(self.amax_m), _ptr(self.amax_v),
            self.m_fmt, self.v_fmt, lr, beta1, beta2, eps, wd, t, flags, _ptr(self.stats))
        if rc != 0:
            raise ValueError("oracle step rejected its arguments (rc=%d)" % rc)
