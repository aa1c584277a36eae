"""The C-ABI library on the host (no GPU needed): it loads, exports every
symbol include/fp8adam.h declares, and rejects bad arguments with error
codes before touching the GPU."""
import ctypes
import os
import re

import pytest

from fp8_quantized_adam_b200 import build as b
from fp8_quantized_adam_b200 import capi

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "fp8adam.h")


@pytest.fixture(scope="module")
def L():
    b.build()
    return capi.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fp8adam_[a-z_0-9]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
    assert sorted(capi.EXPORTED) == names


def test_strerror(L):
    assert capi.fp8adam_strerror(0) == "ok"
    for code in (-1, -2, -3, -4, -5):
        assert capi.fp8adam_strerror(code) not in ("ok", "unknown error")
    assert capi.fp8adam_strerror(-99) == "unknown error"


def test_create_rejects_bad_arguments_on_host(L):
    T = capi.fp8adam_tensor * 1
    out = ctypes.c_void_p()
    t = T(capi.fp8adam_tensor(8, 8, 8, 8, 16))
    # null output / tensors / arrays
    assert L.fp8adam_create(t, 1, 8, 8, 8, 8, 0, 1, 0, None) == capi.ERR_INVALID_ARG
    assert L.fp8adam_create(None, 1, 8, 8, 8, 8, 0, 1, 0, ctypes.byref(out)) == capi.ERR_INVALID_ARG
    assert L.fp8adam_create(t, 1, None, 8, 8, 8, 0, 1, 0, ctypes.byref(out)) == capi.ERR_INVALID_ARG
    assert L.fp8adam_create(t, 0, 8, 8, 8, 8, 0, 1, 0, ctypes.byref(out)) == capi.ERR_INVALID_ARG
    # formats and flags
    assert L.fp8adam_create(t, 1, 8, 8, 8, 8, 3, 1, 0, ctypes.byref(out)) == capi.ERR_UNSUPPORTED_FMT
    assert L.fp8adam_create(t, 1, 8, 8, 8, 8, 0, -1, 0, ctypes.byref(out)) == capi.ERR_UNSUPPORTED_FMT
    assert L.fp8adam_create(t, 1, 8, 8, 8, 8, 0, 1, 64, ctypes.byref(out)) == capi.ERR_INVALID_ARG
    # negative size, null buffer with elements
    bad = T(capi.fp8adam_tensor(8, 8, 8, 8, -1))
    assert L.fp8adam_create(bad, 1, 8, 8, 8, 8, 0, 1, 0, ctypes.byref(out)) == capi.ERR_INVALID_ARG
    bad = T(capi.fp8adam_tensor(8, None, 8, 8, 5))
    assert L.fp8adam_create(bad, 1, 8, 8, 8, 8, 0, 1, 0, ctypes.byref(out)) == capi.ERR_INVALID_ARG
    assert out.value is None


def test_step_and_codec_reject_bad_arguments_on_host(L):
    assert L.fp8adam_step(None, 1e-3, 0.9, 0.95, 1e-8, 0.1, 1, None) == capi.ERR_INVALID_ARG
    assert L.fp8adam_get_stats(None, None, None) == capi.ERR_INVALID_ARG
    assert L.fp8adam_reset_stats(None, None) == capi.ERR_INVALID_ARG
    assert L.fp8adam_destroy(None) == capi.OK
    assert L.fp8adam_encode(2, 8, 8, 4, 0, None) == capi.ERR_UNSUPPORTED_FMT
    assert L.fp8adam_encode(0, 8, 8, 4, 2, None) == capi.ERR_INVALID_ARG
    assert L.fp8adam_encode(0, 8, 8, -1, 0, None) == capi.ERR_INVALID_ARG
    assert L.fp8adam_encode(0, 8, 8, 0, 0, None) == capi.OK  # nothing to do
    assert L.fp8adam_decode(5, 8, 8, 4, 0, None) == capi.ERR_UNSUPPORTED_FMT
    assert L.fp8adam_encode_bits_range(0, 0xFFFFFFFF, 2, 16, 0, None) == capi.ERR_INVALID_ARG
    assert L.fp8adam_encode_bits_range(0, 0, 4, 2, 0, None) == capi.ERR_INVALID_ARG  # misaligned out
    assert L.fp8adam_encode_sr(2, 8, 8, 8, 4, None) == capi.ERR_UNSUPPORTED_FMT
    assert L.fp8adam_encode_sr(0, 8, 8, 8, -1, None) == capi.ERR_INVALID_ARG
    assert L.fp8adam_encode_sr(0, None, 8, 8, 4, None) == capi.ERR_INVALID_ARG
    assert L.fp8adam_encode_sr(1, 8, None, 8, 4, None) == capi.ERR_INVALID_ARG
    assert L.fp8adam_encode_sr(0, 8, 8, 8, 0, None) == capi.OK  # nothing to do
    assert isinstance(capi.fp8adam_launch_count(), int)


def test_binding_raises_on_error_codes(L):
    with pytest.raises(capi.Fp8AdamError) as e:
        capi.fp8adam_step(0, 1e-3, 0.9, 0.95, 1e-8, 0.1, 1, 0)
    assert e.value.code == capi.ERR_INVALID_ARG


def test_create_rejects_overlapping_written_buffers_on_host(L):
    """Checked before any CUDA call: fake addresses suffice.  A written buffer
    (param, m, v) overlapping any other is OVERLAP; gradients may alias one
    another; disjoint buffers get past the check (and then fail with CUDA on
    a machine without a GPU, or succeed on one with a GPU)."""
    T = capi.fp8adam_tensor
    base = 1 << 32

    def create(specs):
        arr = (T * len(specs))(*[T(*x) for x in specs])
        out = ctypes.c_void_p()
        rc = L.fp8adam_create(arr, len(specs), 8, 8, 8, 8, 0, 1, 0, ctypes.byref(out))
        if rc == capi.OK:  # a GPU is present: nothing was launched, just free the tables
            L.fp8adam_destroy(out)
        return rc

    n = 1000
    t0 = (base, base + 0x10000, base + 0x20000, base + 0x30000, n)
    assert create([t0, t0]) == capi.ERR_OVERLAP                       # the same tensor twice
    t1 = (base + 4 * n - 4, base + 0x40000, base + 0x50000, base + 0x60000, n)
    assert create([t0, t1]) == capi.ERR_OVERLAP                       # params overlap by 4 bytes
    t2 = (base + 0x70000, base + 0x10000, base + 0x80000, base + 0x90000, n)
    assert create([t0, t2]) != capi.ERR_OVERLAP                       # shared gradient buffer: read only
    t3 = (base + 0x70000, base + 0x80000, base + 0x90000, base + 0x10000 + 10, n)
    assert create([t0, t3]) == capi.ERR_OVERLAP                       # a v written over a gradient
    t4 = (base + 4 * n, base + 0xA0000, base + 0xB0000, base + 0xC0000, n)
    assert create([t0, t4]) != capi.ERR_OVERLAP                       # adjacent, not overlapping
    assert create([t0, (base, base, base, base, 0)]) != capi.ERR_OVERLAP  # an empty tensor has no bytes
    assert create([(base, base + 8, base + 16, base + 24, (1 << 48) + 1)]) == capi.ERR_INVALID_ARG  # size bound


def test_schedule_entry_points_reject_bad_arguments_on_host(L):
    sp = (capi.fp8adam_step_params * 1)(capi.fp8adam_step_params(1e-3, 0.9, 0.95, 1e-8, 0.1, 2, 1.0, 0.0, 0))
    assert L.fp8adam_set_schedule(None, sp, 1, None) == capi.ERR_INVALID_ARG
    assert L.fp8adam_step_scheduled(None, None) == capi.ERR_INVALID_ARG
    t = ctypes.c_int64(0)
    assert L.fp8adam_get_schedule_step(None, ctypes.byref(t), None) == capi.ERR_INVALID_ARG
    assert L.fp8adam_strerror(capi.ERR_SCHEDULE_END).startswith(b"a scheduled step")


def test_release_build_has_no_debug_hooks(L):
    assert L.fp8adam_debug_inject_wait(0, 1) == capi.ERR_INVALID_ARG
    assert L.fp8adam_debug_set_numel(None, 0, 0) == capi.ERR_INVALID_ARG


def test_debug_build_loads_and_exports_the_same_symbols(L):
    D = capi.debug_lib()
    for name in capi.EXPORTED:
        assert hasattr(D, name), name
    assert D.fp8adam_debug_set_numel(None, 0, 0) == capi.ERR_INVALID_ARG  # host-side check, no GPU
    assert D.fp8adam_strerror(capi.ERR_DEBUG_BOUNDS).startswith(b"a kernel access")


def test_host_step_rejects_bad_arguments_on_host(L):
    sp = capi.fp8adam_step_params(1e-3, 0.9, 0.95, 1e-8, 0.1, 1, 1.0, 0.0, 0)
    ptrs = (ctypes.c_void_p * 1)()
    assert L.fp8adam_step_host(None, ctypes.byref(sp), ptrs, None, None) == capi.ERR_INVALID_ARG
    assert L.fp8adam_step_host(None, None, ptrs, None, None) == capi.ERR_INVALID_ARG


def test_option_entry_points_reject_bad_arguments_on_host(L):
    T = capi.fp8adam_tensor * 1
    t = T(capi.fp8adam_tensor(8, 8, 8, 8, 16))
    out = ctypes.c_void_p()
    ok = dict(scale_m=8, scale_v=8, amax_m=8, amax_v=8, m_fmt=0, v_fmt=1)
    assert L.fp8adam_create_ex(t, 1, None, ctypes.byref(out)) == capi.ERR_INVALID_ARG
    for bad in (dict(margin_m=-1), dict(margin_v=65), dict(amax_history_len=4), dict(amax_history_len=2000),
                dict(flags=64), dict(flags=capi.FLAG_SR_DRAW16), dict(scale_v=0), dict(chunk_elems=100), dict(chunk_elems=1 << 20),
                dict(chunk_elems=-4096)):
        o = capi.fp8adam_options(**{**ok, **bad})
        assert L.fp8adam_create_ex(t, 1, ctypes.byref(o), ctypes.byref(out)) == capi.ERR_INVALID_ARG, bad
    o = capi.fp8adam_options(**{**ok, "m_fmt": 7})
    assert L.fp8adam_create_ex(t, 1, ctypes.byref(o), ctypes.byref(out)) == capi.ERR_UNSUPPORTED_FMT
    sp = capi.fp8adam_step_params(1e-3, 0.9, 0.95, 1e-8, 0.1, 1, 1.0, 0.0, 0)
    assert L.fp8adam_step_ex(None, ctypes.byref(sp), None) == capi.ERR_INVALID_ARG
    assert L.fp8adam_get_grad_info(None, None, None, None) == capi.ERR_INVALID_ARG
    assert L.fp8adam_check(None, None) == capi.ERR_INVALID_ARG
    assert "not usable" in capi.fp8adam_strerror(capi.ERR_DEVICE_TIMEOUT)
