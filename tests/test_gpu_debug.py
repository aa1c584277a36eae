"""The debug build (libfp8adam_debug.so, compiled with FP8ADAM_DEBUG), through
its C ABI:
- with every global access bounds-checked it gives the release build's
  results bit for bit and reports no violation;
- a staged kernel's bounded wait made to run out (one CTA's copies are never
  issued: a barrier that nothing completes) ends the kernel with
  FP8ADAM_ERR_DEVICE_TIMEOUT, without a fault, and the context then runs
  normal steps again;
- a tensor table that under-states a tensor's size makes the bounds checks
  skip the accesses past it and report FP8ADAM_ERR_DEBUG_BOUNDS (every access
  stays inside the real buffers)."""
import ctypes
import time

import pytest
import torch

from fp8_quantized_adam_b200 import capi, workloads
from gpu_harness import HP

pytestmark = pytest.mark.gpu

SIZES = [70001, 4096, 33, 0, 3 * 4096 + 5, 200003]
SEED = 51


class Model:
    """The C ABI on a seeded model; `opts` (fp8adam_options fields) creates
    the context with fp8adam_create_ex."""

    def __init__(self, L, opts=None):
        self.L = L
        self.specs = workloads.custom_layout(SIZES)
        self.M = workloads.FlatModel(self.specs, torch.device("cuda:0"))
        self.sig = workloads.tensor_sigmas(self.specs, SEED)
        self.reset()
        M = self.M
        arr = (capi.fp8adam_tensor * M.T)()
        for i in range(M.T):
            arr[i] = capi.fp8adam_tensor(M.view(M.p, i).data_ptr(), M.view(M.g, i).data_ptr(),
                                         M.view(M.m, i).data_ptr(), M.view(M.v, i).data_ptr(), self.specs[i].numel)
        out = ctypes.c_void_p()
        if opts is None:
            assert L.fp8adam_create(arr, M.T, M.scale_m.data_ptr(), M.scale_v.data_ptr(), M.amax_m.data_ptr(),
                                    M.amax_v.data_ptr(), 0, 1, 0, ctypes.byref(out)) == capi.OK
        else:
            kw = dict(opts)
            self.keep = []  # host arrays and device buffers the options point to
            if kw.get("amax_history_len", 0) > 1:
                h = torch.zeros(2, kw["amax_history_len"], M.T, device="cuda:0")
                self.keep.append(h)
                kw["amax_history_m"], kw["amax_history_v"] = h[0].data_ptr(), h[1].data_ptr()
            if "sr_counter_ids" in kw:
                ids = (ctypes.c_uint32 * M.T)(*kw["sr_counter_ids"])
                self.keep.append(ids)
                kw["sr_counter_ids"] = ctypes.cast(ids, ctypes.c_void_p)
            o = capi.fp8adam_options(scale_m=M.scale_m.data_ptr(), scale_v=M.scale_v.data_ptr(),
                                     amax_m=M.amax_m.data_ptr(), amax_v=M.amax_v.data_ptr(), m_fmt=0, v_fmt=1, **kw)
            assert L.fp8adam_create_ex(arr, M.T, ctypes.byref(o), ctypes.byref(out)) == capi.OK
        self.ctx = out
        self.stream = torch.cuda.current_stream().cuda_stream

    def reset(self):
        M = self.M
        workloads.init_params_into(self.specs, M.views(M.p), SEED)
        for x in (M.m, M.v, M.amax_m, M.amax_v):
            x.zero_()
        M.scale_m.fill_(1.0)
        M.scale_v.fill_(1.0)

    def step(self, t):
        workloads.grads_into(self.specs, self.M.views(self.M.g), SEED, t, self.sig)
        return self.L.fp8adam_step(self.ctx, HP["lr"], HP["beta1"], HP["beta2"], HP["eps"], HP["weight_decay"], t,
                                   self.stream)

    def check(self):
        return self.L.fp8adam_check(self.ctx, self.stream)

    def state(self):
        torch.cuda.synchronize()
        M = self.M
        return [x.clone() for x in (M.p, M.m, M.v, M.scale_m, M.scale_v, M.amax_m, M.amax_v)]

    def close(self):
        torch.cuda.synchronize()
        self.L.fp8adam_destroy(self.ctx)


def _same(a, b):
    return all(torch.equal(x.view(torch.uint8), y.view(torch.uint8)) for x, y in zip(a, b))


def _release_state(steps, opts=None):
    r = Model(capi.lib(), opts)
    for t in range(1, steps + 1):
        assert r.step(t) == capi.OK
    assert r.check() == capi.OK
    s = r.state()
    r.close()
    return s


def test_debug_build_matches_release_and_reports_nothing():
    want = _release_state(4)
    d = Model(capi.debug_lib())
    for t in range(1, 5):
        assert d.step(t) == capi.OK
    assert d.check() == capi.OK
    assert _same(d.state(), want)
    d.close()


@pytest.mark.parametrize("opts", [
    dict(flags=capi.FLAG_STOCHASTIC_ROUNDING | capi.FLAG_SR_DRAW16, seed=9, sr_counter_ids=[5, 1, 9, 2, 7, 3]),
    dict(flags=capi.FLAG_STOCHASTIC_ROUNDING, seed=9, amax_history_len=3, margin_m=1, margin_v=2)],
    ids=["sr16_ids", "sr32_history_margin"])
def test_debug_build_matches_release_with_options(opts):
    """The option kernels (stochastic rounding with 16-bit draws and counter
    ids; with 32-bit draws, an amax history and margins) in the debug build:
    the release build's results bit for bit, and no bounds violation."""
    want = _release_state(4, opts)
    d = Model(capi.debug_lib(), opts)
    for t in range(1, 5):
        assert d.step(t) == capi.OK
    assert d.check() == capi.OK
    assert _same(d.state(), want)
    d.close()


def test_bounded_wait_runs_out_and_the_context_recovers():
    L = capi.debug_lib()
    d = Model(L)
    # CTA 0 runs the first chunk of the 70001-element tensor: 8 sub-tiles of
    # 2048; its sub-tile 1 is armed but never filled
    assert L.fp8adam_debug_inject_wait(0, 1) == capi.OK
    try:
        t0 = time.perf_counter()
        assert d.step(1) == capi.OK
        rc = d.check()
        waited = time.perf_counter() - t0
    finally:
        assert L.fp8adam_debug_inject_wait(-1, -1) == capi.OK
    assert rc == capi.ERR_DEVICE_TIMEOUT
    assert waited < 120.0
    print("bounded wait ran out after %.2f s" % waited)
    assert d.check() == capi.OK  # the error word was cleared
    # the context runs normal steps again: from a fresh state, the release results
    d.reset()
    for t in range(1, 5):
        assert d.step(t) == capi.OK
    assert d.check() == capi.OK
    assert _same(d.state(), _release_state(4))
    d.close()


def test_bounds_checks_skip_accesses_past_a_tensor():
    L = capi.debug_lib()
    d = Model(L)
    assert d.step(1) == capi.OK
    assert d.check() == capi.OK
    assert L.fp8adam_debug_set_numel(d.ctx, 0, 1000) == capi.OK  # the table now under-states tensor 0
    assert d.step(2) == capi.OK
    assert d.check() == capi.ERR_DEBUG_BOUNDS
    assert L.fp8adam_debug_set_numel(d.ctx, 0, SIZES[0] + 1) == capi.ERR_INVALID_ARG  # never above the real size
    assert L.fp8adam_debug_set_numel(d.ctx, 0, SIZES[0]) == capi.OK
    d.reset()
    for t in range(1, 5):
        assert d.step(t) == capi.OK
    assert d.check() == capi.OK
    assert _same(d.state(), _release_state(4))
    d.close()
