"""ctypes binding of ``libfp8adam.so`` (C ABI in include/fp8adam.h).

Argument marshalling only: every function forwards to the C entry point of
the same name, and every step of the optimizer runs in the library's CUDA
kernels.  There is no fallback: if the library is missing, loading raises.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfp8adam.so")
DEBUG_LIB_PATH = os.path.join(_PKG, "libfp8adam_debug.so")

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED_FMT = -2
ERR_CUDA = -3
ERR_OOM = -4
ERR_WRONG_DEVICE = -5
ERR_NOALLOC_LIMIT = -6
ERR_DEVICE_TIMEOUT = -7
ERR_DEBUG_BOUNDS = -8
ERR_OVERLAP = -9
ERR_SCHEDULE_END = -10
NOALLOC_MAX_TENSORS = 4096

E4M3, E5M2, FP32 = 0, 1, 2
FLAG_STATS = 1
FLAG_JIT_EVERY_STEP = 2
FLAG_UPDATE_FROM_STORED = 4
FLAG_STOCHASTIC_ROUNDING = 8
FLAG_SR_DRAW16 = 32  # with FLAG_STOCHASTIC_ROUNDING: 16-bit draws, hardware conversion
FLAG_NO_TMA = 16


class fp8adam_tensor(ctypes.Structure):
    _fields_ = [("param", ctypes.c_void_p), ("grad", ctypes.c_void_p), ("m", ctypes.c_void_p),
                ("v", ctypes.c_void_p), ("numel", ctypes.c_int64)]


class fp8adam_options(ctypes.Structure):
    _fields_ = [("scale_m", ctypes.c_void_p), ("scale_v", ctypes.c_void_p), ("amax_m", ctypes.c_void_p),
                ("amax_v", ctypes.c_void_p), ("m_fmt", ctypes.c_int32), ("v_fmt", ctypes.c_int32),
                ("flags", ctypes.c_uint32), ("margin_m", ctypes.c_int32), ("margin_v", ctypes.c_int32),
                ("amax_history_len", ctypes.c_int32), ("amax_history_m", ctypes.c_void_p),
                ("amax_history_v", ctypes.c_void_p), ("seed", ctypes.c_uint64), ("param_bf16", ctypes.c_void_p),
                ("chunk_elems", ctypes.c_int32), ("sr_counter_ids", ctypes.c_void_p)]


class fp8adam_step_params(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("weight_decay", ctypes.c_float), ("step", ctypes.c_int64),
                ("loss_scale", ctypes.c_float), ("max_norm", ctypes.c_float), ("skip_nonfinite", ctypes.c_int32)]


class Fp8AdamError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__("%s failed: %s (%d)" % (fn, fp8adam_strerror(code), code))
        self.code = code


_lib = None
_debug_lib = None


def lib() -> ctypes.CDLL:
    """Load the CUDA library; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libfp8adam.so is not built (python -m fp8_quantized_adam_b200.build)")
        _lib = _bind(ctypes.CDLL(LIB_PATH))
    return _lib


def debug_lib() -> ctypes.CDLL:
    """The debug build (bounds checks that report FP8ADAM_ERR_DEBUG_BOUNDS,
    the bounded-wait injection point), same C ABI; for tests."""
    global _debug_lib
    if _debug_lib is None:
        if not os.path.exists(DEBUG_LIB_PATH):
            raise RuntimeError("libfp8adam_debug.so is not built (python -m fp8_quantized_adam_b200.build)")
        _debug_lib = _bind(ctypes.CDLL(DEBUG_LIB_PATH))
    return _debug_lib


def _bind(L: ctypes.CDLL) -> ctypes.CDLL:
    """Argument and result types of every exported call."""
    vp, i32, i64, u32, f = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32, ctypes.c_float
    L.fp8adam_create.restype = ctypes.c_int
    L.fp8adam_create.argtypes = [ctypes.POINTER(fp8adam_tensor), i32, vp, vp, vp, vp, i32, i32, u32,
                                 ctypes.POINTER(vp)]
    L.fp8adam_step.restype = ctypes.c_int
    L.fp8adam_step.argtypes = [vp, f, f, f, f, f, i64, vp]
    L.fp8adam_get_stats.restype = ctypes.c_int
    L.fp8adam_get_stats.argtypes = [vp, ctypes.POINTER(ctypes.c_uint64), vp]
    L.fp8adam_reset_stats.restype = ctypes.c_int
    L.fp8adam_reset_stats.argtypes = [vp, vp]
    L.fp8adam_destroy.restype = ctypes.c_int
    L.fp8adam_destroy.argtypes = [vp]
    L.fp8adam_strerror.restype = ctypes.c_char_p
    L.fp8adam_strerror.argtypes = [ctypes.c_int]
    L.fp8adam_encode.restype = ctypes.c_int
    L.fp8adam_encode.argtypes = [i32, vp, vp, i64, i32, vp]
    L.fp8adam_encode_bits_range.restype = ctypes.c_int
    L.fp8adam_encode_bits_range.argtypes = [i32, u32, i64, vp, i32, vp]
    L.fp8adam_decode.restype = ctypes.c_int
    L.fp8adam_decode.argtypes = [i32, vp, vp, i64, i32, vp]
    L.fp8adam_step_host.restype = ctypes.c_int
    L.fp8adam_step_host.argtypes = [vp, ctypes.POINTER(fp8adam_step_params), ctypes.POINTER(ctypes.c_void_p),
                                    vp, vp]
    L.fp8adam_encode_sr.restype = ctypes.c_int
    L.fp8adam_encode_sr.argtypes = [i32, vp, vp, vp, i64, vp]
    L.fp8adam_encode_sr16.restype = ctypes.c_int
    L.fp8adam_encode_sr16.argtypes = [i32, vp, vp, vp, i64, vp]
    L.fp8adam_launch_count.restype = ctypes.c_uint64
    L.fp8adam_launch_count.argtypes = []
    L.fp8adam_create_ex.restype = ctypes.c_int
    L.fp8adam_create_ex.argtypes = [ctypes.POINTER(fp8adam_tensor), i32, ctypes.POINTER(fp8adam_options),
                                    ctypes.POINTER(vp)]
    L.fp8adam_step_ex.restype = ctypes.c_int
    L.fp8adam_step_ex.argtypes = [vp, ctypes.POINTER(fp8adam_step_params), vp]
    L.fp8adam_check.restype = ctypes.c_int
    L.fp8adam_check.argtypes = [vp, vp]
    L.fp8adam_get_grad_info.restype = ctypes.c_int
    L.fp8adam_get_grad_info.argtypes = [vp, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_uint32), vp]
    L.fp8adam_step_noalloc.restype = ctypes.c_int
    L.fp8adam_step_noalloc.argtypes = [ctypes.POINTER(fp8adam_tensor), i32, vp, vp, vp, vp, i32, i32, u32,
                                       f, f, f, f, f, i64, vp]
    L.fp8adam_set_schedule.restype = ctypes.c_int
    L.fp8adam_set_schedule.argtypes = [vp, ctypes.POINTER(fp8adam_step_params), i32, vp]
    L.fp8adam_step_scheduled.restype = ctypes.c_int
    L.fp8adam_step_scheduled.argtypes = [vp, vp]
    L.fp8adam_get_schedule_step.restype = ctypes.c_int
    L.fp8adam_get_schedule_step.argtypes = [vp, ctypes.POINTER(ctypes.c_int64), vp]
    L.fp8adam_debug_inject_wait.restype = ctypes.c_int
    L.fp8adam_debug_inject_wait.argtypes = [i32, i32]
    L.fp8adam_debug_set_numel.restype = ctypes.c_int
    L.fp8adam_debug_set_numel.argtypes = [vp, i32, i64]
    return L


def _check(fn: str, rc: int) -> int:
    if rc != OK:
        raise Fp8AdamError(fn, rc)
    return rc


# ---- the C entry points, same names --------------------------------------
def fp8adam_strerror(code: int) -> str:
    return lib().fp8adam_strerror(code).decode()


def fp8adam_create(tensors, num_tensors: int, scale_m: int, scale_v: int, amax_m: int, amax_v: int,
                   m_fmt: int, v_fmt: int, flags: int) -> int:
    """tensors: a ctypes array of fp8adam_tensor; pointers are ints.
    Returns the context handle (int)."""
    out = ctypes.c_void_p()
    _check("fp8adam_create", lib().fp8adam_create(tensors, num_tensors, scale_m, scale_v, amax_m, amax_v,
                                                  m_fmt, v_fmt, flags, ctypes.byref(out)))
    return out.value


def fp8adam_create_ex(tensors, num_tensors: int, opts: fp8adam_options) -> int:
    out = ctypes.c_void_p()
    _check("fp8adam_create_ex", lib().fp8adam_create_ex(tensors, num_tensors, ctypes.byref(opts), ctypes.byref(out)))
    return out.value


def fp8adam_step_ex(ctx: int, params: fp8adam_step_params, cuda_stream: int) -> None:
    _check("fp8adam_step_ex", lib().fp8adam_step_ex(ctx, ctypes.byref(params), cuda_stream))


def fp8adam_get_grad_info(ctx: int, cuda_stream: int):
    n = ctypes.c_double()
    k = ctypes.c_uint32()
    _check("fp8adam_get_grad_info", lib().fp8adam_get_grad_info(ctx, ctypes.byref(n), ctypes.byref(k), cuda_stream))
    return n.value, int(k.value)


def fp8adam_step(ctx: int, lr: float, beta1: float, beta2: float, eps: float, weight_decay: float,
                 step: int, cuda_stream: int) -> None:
    _check("fp8adam_step", lib().fp8adam_step(ctx, lr, beta1, beta2, eps, weight_decay, step, cuda_stream))


def fp8adam_get_stats(ctx: int, cuda_stream: int):
    out = (ctypes.c_uint64 * 2)()
    _check("fp8adam_get_stats", lib().fp8adam_get_stats(ctx, out, cuda_stream))
    return int(out[0]), int(out[1])


def fp8adam_reset_stats(ctx: int, cuda_stream: int) -> None:
    _check("fp8adam_reset_stats", lib().fp8adam_reset_stats(ctx, cuda_stream))


def fp8adam_check(ctx: int, cuda_stream: int) -> None:
    _check("fp8adam_check", lib().fp8adam_check(ctx, cuda_stream))


def fp8adam_destroy(ctx: int) -> None:
    _check("fp8adam_destroy", lib().fp8adam_destroy(ctx))


def fp8adam_encode(fmt: int, x: int, out: int, n: int, impl: int, cuda_stream: int) -> None:
    _check("fp8adam_encode", lib().fp8adam_encode(fmt, x, out, n, impl, cuda_stream))


def fp8adam_encode_bits_range(fmt: int, first: int, n: int, out: int, impl: int, cuda_stream: int) -> None:
    _check("fp8adam_encode_bits_range", lib().fp8adam_encode_bits_range(fmt, first, n, out, impl, cuda_stream))


def fp8adam_step_host(ctx, params: fp8adam_step_params, host_grads, amax_host: int, cuda_stream: int) -> None:
    """host_grads: a ctypes array of host pointers, one per tensor."""
    _check("fp8adam_step_host", lib().fp8adam_step_host(ctx, ctypes.byref(params), host_grads, amax_host or None,
                                                        cuda_stream))


def fp8adam_set_schedule(ctx, steps, cuda_stream: int) -> None:
    """steps: a sequence of fp8adam_step_params for consecutive steps."""
    arr = (fp8adam_step_params * len(steps))(*steps)
    _check("fp8adam_set_schedule", lib().fp8adam_set_schedule(ctx, arr, len(steps), cuda_stream))


def fp8adam_step_scheduled(ctx, cuda_stream: int) -> None:
    _check("fp8adam_step_scheduled", lib().fp8adam_step_scheduled(ctx, cuda_stream))


def fp8adam_get_schedule_step(ctx, cuda_stream: int) -> int:
    t = ctypes.c_int64(0)
    _check("fp8adam_get_schedule_step", lib().fp8adam_get_schedule_step(ctx, ctypes.byref(t), cuda_stream))
    return int(t.value)


def fp8adam_encode_sr(fmt: int, x: int, r: int, out: int, n: int, cuda_stream: int) -> None:
    _check("fp8adam_encode_sr", lib().fp8adam_encode_sr(fmt, x, r, out, n, cuda_stream))


def fp8adam_encode_sr16(fmt: int, x: int, w: int, out: int, n: int, cuda_stream: int) -> None:
    _check("fp8adam_encode_sr16", lib().fp8adam_encode_sr16(fmt, x, w, out, n, cuda_stream))


def fp8adam_decode(fmt: int, codes: int, out: int, n: int, impl: int, cuda_stream: int) -> None:
    _check("fp8adam_decode", lib().fp8adam_decode(fmt, codes, out, n, impl, cuda_stream))


def fp8adam_launch_count() -> int:
    return int(lib().fp8adam_launch_count())


def fp8adam_step_noalloc(tensors, num_tensors: int, scale_m: int, scale_v: int, amax_m: int, amax_v: int,
                         m_fmt: int, v_fmt: int, flags: int, lr: float, beta1: float, beta2: float,
                         eps: float, weight_decay: float, step: int, cuda_stream: int) -> None:
    """The allocation-free step (see include/fp8adam.h): for callers that
    cannot allocate device memory; uses the library's fixed scratch array."""
    _check("fp8adam_step_noalloc", lib().fp8adam_step_noalloc(
        tensors, num_tensors, scale_m, scale_v, amax_m, amax_v, m_fmt, v_fmt, flags, lr, beta1, beta2,
        eps, weight_decay, step, cuda_stream))


EXPORTED = ["fp8adam_create", "fp8adam_step", "fp8adam_get_stats", "fp8adam_reset_stats",
            "fp8adam_destroy", "fp8adam_strerror", "fp8adam_encode", "fp8adam_encode_bits_range",
            "fp8adam_decode", "fp8adam_launch_count", "fp8adam_step_noalloc", "fp8adam_create_ex",
            "fp8adam_step_ex", "fp8adam_get_grad_info", "fp8adam_check", "fp8adam_encode_sr", "fp8adam_encode_sr16",
            "fp8adam_step_host",
            "fp8adam_debug_inject_wait", "fp8adam_debug_set_numel", "fp8adam_set_schedule",
            "fp8adam_step_scheduled", "fp8adam_get_schedule_step"]
