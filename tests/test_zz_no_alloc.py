"""The allocation-free step, fp8adam_step_noalloc, through the C ABI.

Some callers cannot allocate device memory: a custom allocator or memory-pool
callback, a framework hook that must not grow the footprint, a process whose
memory is reserved up front.  fp8adam_step_noalloc serves them with the
library's own fixed scratch array instead of the buffers fp8adam_create
allocates.  These tests check that two calls in a row give exactly what the
regular entry points give on identical inputs (non-finite gradients
included), and that overlapping buffers and a tensor list larger than the
scratch holds are refused.  The file is named to be collected last,
and each test builds all its inputs itself, so it passes alone in a fresh
process as well as after the other tests.
"""
import numpy as np
import pytest
import torch

from fp8_quantized_adam_b200 import FP8AdamW, capi, workloads

pytestmark = pytest.mark.gpu

HP = workloads.HPARAMS
SIZES = [70001, 4096, 17, 0, 2 * 65536 + 3, 1 << 20]


def _model(cfg):
    specs = workloads.custom_layout(SIZES)
    m = workloads.FlatModel(specs, torch.device("cuda:0"))
    workloads.init_params_into(specs, m.views(m.p), cfg)
    return specs, m


def _tensor_array(m):
    T = m.T
    arr = (capi.fp8adam_tensor * T)()
    for i in range(T):
        arr[i] = capi.fp8adam_tensor(m.view(m.p, i).data_ptr(), m.view(m.g, i).data_ptr(),
                                     m.view(m.m, i).data_ptr(), m.view(m.v, i).data_ptr(),
                                     m.specs[i].numel)
    return arr


@pytest.mark.parametrize("jit_every_step", [False, True], ids=["delayed", "current"])
def test_noalloc_matches_regular_step_two_calls(jit_every_step):
    cfg = 31
    specs, ref = _model(cfg)
    _, na = _model(cfg)
    sig = workloads.tensor_sigmas(specs, cfg)
    opt = FP8AdamW(ref.views(ref.p), ref.views(ref.g), m=ref.views(ref.m), v=ref.views(ref.v),
                   scale_m=ref.scale_m, scale_v=ref.scale_v, amax_m=ref.amax_m, amax_v=ref.amax_v,
                   jit_every_step=jit_every_step)
    arr = _tensor_array(na)
    flags = capi.FLAG_JIT_EVERY_STEP if jit_every_step else 0
    stream = torch.cuda.current_stream().cuda_stream
    for t in (1, 2):  # two calls in a row
        workloads.grads_into(specs, ref.views(ref.g), cfg, t, sig)
        na.g.copy_(ref.g)
        opt.step()
        capi.fp8adam_step_noalloc(arr, na.T, na.scale_m.data_ptr(), na.scale_v.data_ptr(),
                                  na.amax_m.data_ptr(), na.amax_v.data_ptr(), capi.E4M3, capi.E5M2, flags,
                                  HP["lr"], HP["beta1"], HP["beta2"], HP["eps"], HP["weight_decay"], t, stream)
        torch.cuda.synchronize()
        # codes, scales and amax bit for bit; params within the 1e-6 relative
        # tolerance of the parity tests (identical arithmetic: expected exact)
        for name in ("m", "v", "scale_m", "scale_v", "amax_m", "amax_v"):
            assert torch.equal(getattr(ref, name).view(torch.uint8), getattr(na, name).view(torch.uint8)), (t, name)
        p_ref, p_na = ref.p.cpu().numpy().astype(np.float64), na.p.cpu().numpy().astype(np.float64)
        assert (np.abs(p_na - p_ref) <= 1e-6 * np.abs(p_ref)).all(), t
    opt.close()


def test_noalloc_nan_and_inf_gradients_match_regular_step():
    """A NaN and an inf gradient: the amax bits (the canonical NaN where a
    moment is NaN), scales, codes and params equal the regular step's, over
    two calls in a row."""
    cfg = 32
    specs, ref = _model(cfg)
    _, na = _model(cfg)
    sig = workloads.tensor_sigmas(specs, cfg)
    opt = FP8AdamW(ref.views(ref.p), ref.views(ref.g), m=ref.views(ref.m), v=ref.views(ref.v),
                   scale_m=ref.scale_m, scale_v=ref.scale_v, amax_m=ref.amax_m, amax_v=ref.amax_v)
    arr = _tensor_array(na)
    stream = torch.cuda.current_stream().cuda_stream
    for t in (1, 2):
        workloads.grads_into(specs, ref.views(ref.g), cfg, t, sig)
        ref.view(ref.g, 0)[5] = float("nan")
        ref.view(ref.g, 4)[70000] = float("inf")
        na.g.copy_(ref.g)
        opt.step()
        capi.fp8adam_step_noalloc(arr, na.T, na.scale_m.data_ptr(), na.scale_v.data_ptr(),
                                  na.amax_m.data_ptr(), na.amax_v.data_ptr(), capi.E4M3, capi.E5M2, 0,
                                  HP["lr"], HP["beta1"], HP["beta2"], HP["eps"], HP["weight_decay"], t, stream)
        torch.cuda.synchronize()
        assert int(na.amax_m.view(torch.int32)[0]) == 0x7FFFFFFF  # canonical NaN
        for name in ("m", "v", "scale_m", "scale_v", "amax_m", "amax_v"):
            assert torch.equal(getattr(ref, name).view(torch.uint8), getattr(na, name).view(torch.uint8)), (t, name)
        p_ref, p_na = ref.p.cpu().numpy(), na.p.cpu().numpy()
        nan = np.isnan(p_ref)
        assert (np.isnan(p_na) == nan).all()
        assert (np.abs(p_na[~nan].astype(np.float64) - p_ref[~nan]) <= 1e-6 * np.abs(p_ref[~nan])).all(), t
    opt.close()


def test_noalloc_refuses_overlapping_written_buffers():
    """As fp8adam_create: a param range that overlaps another tensor's m
    codes is refused, nothing is queued and the buffers are untouched."""
    dev = torch.device("cuda:0")
    buf = torch.zeros(4096, dtype=torch.uint8, device=dev)
    p = torch.zeros(512, device=dev)
    g = torch.zeros(512, dtype=torch.bfloat16, device=dev)
    arr = (capi.fp8adam_tensor * 2)()
    arr[0] = capi.fp8adam_tensor(p.data_ptr(), g.data_ptr(), buf.data_ptr(), buf.data_ptr() + 1024, 512)
    # tensor 1's param overlaps tensor 0's m codes
    arr[1] = capi.fp8adam_tensor(buf.data_ptr() + 256, g.data_ptr(), buf.data_ptr() + 2048,
                                 buf.data_ptr() + 3072, 16)
    ones = torch.ones(2, device=dev)
    zeros = torch.zeros(2, device=dev)
    with pytest.raises(capi.Fp8AdamError) as e:
        capi.fp8adam_step_noalloc(arr, 2, ones.data_ptr(), ones.data_ptr(), zeros.data_ptr(), zeros.data_ptr(),
                                  capi.E4M3, capi.E5M2, 0, 1e-3, 0.9, 0.95, 1e-8, 0.0, 1,
                                  torch.cuda.current_stream().cuda_stream)
    assert e.value.code == capi.ERR_OVERLAP
    torch.cuda.synchronize()
    assert int(buf.sum()) == 0 and float(p.abs().sum()) == 0.0


def test_noalloc_refuses_more_tensors_than_its_scratch_holds():
    n = capi.NOALLOC_MAX_TENSORS + 1
    buf = torch.zeros(64, device="cuda:0")
    arr = (capi.fp8adam_tensor * n)()
    for i in range(n):
        arr[i] = capi.fp8adam_tensor(buf.data_ptr(), buf.data_ptr(), buf.data_ptr(), buf.data_ptr(), 0)
    ones = torch.ones(n, device="cuda:0")
    with pytest.raises(capi.Fp8AdamError) as e:
        capi.fp8adam_step_noalloc(arr, n, ones.data_ptr(), ones.data_ptr(), ones.data_ptr(), ones.data_ptr(),
                                  capi.E4M3, capi.E5M2, 0, 1e-3, 0.9, 0.95, 1e-8, 0.0, 1,
                                  torch.cuda.current_stream().cuda_stream)
    assert e.value.code == capi.ERR_NOALLOC_LIMIT
    assert "FP8ADAM_NOALLOC_MAX_TENSORS" in capi.fp8adam_strerror(capi.ERR_NOALLOC_LIMIT)
