"""Scheduled steps (fp8adam_set_schedule / fp8adam_step_scheduled): the step's
constants come from a device schedule, so one captured launch sequence can be
replayed as a CUDA graph.  Checked: a learning-rate schedule against the oracle
bit for bit; a captured and replayed step against the regular step path; the
option kernels; current scaling from step 1; running past the end."""
import numpy as np
import pytest
import torch

import oracle
from fp8_quantized_adam_b200 import FP8AdamW, capi, workloads
from gpu_harness import HP, bf16_host_bits

pytestmark = pytest.mark.gpu

SIZES = [70001, 4096, 33, 0, 3 * 4096 + 5, 200003]
LRS = [3e-4, 2.5e-4, 1e-4, 5e-5, 1e-5, 7e-4]


class Twin:
    """A model and its optimizer on seeded inputs."""

    def __init__(self, cfg, **opt):
        self.specs = workloads.custom_layout(SIZES)
        self.M = workloads.FlatModel(self.specs, torch.device("cuda:0"))
        workloads.init_params_into(self.specs, self.M.views(self.M.p), cfg)
        self.cfg = cfg
        self.sig = workloads.tensor_sigmas(self.specs, cfg)
        M = self.M
        self.opt = FP8AdamW(M.views(M.p), M.views(M.g), m=M.views(M.m), v=M.views(M.v), scale_m=M.scale_m,
                            scale_v=M.scale_v, amax_m=M.amax_m, amax_v=M.amax_v, lr=HP["lr"],
                            betas=(HP["beta1"], HP["beta2"]), eps=HP["eps"], weight_decay=HP["weight_decay"], **opt)

    def grads(self, t):
        workloads.grads_into(self.specs, self.M.views(self.M.g), self.cfg, t, self.sig)

    def state(self):
        torch.cuda.synchronize()
        M = self.M
        return [x.clone() for x in (M.p, M.m, M.v, M.scale_m, M.scale_v, M.amax_m, M.amax_v)]


def _same(a, b):
    return all(torch.equal(x.view(torch.uint8), y.view(torch.uint8)) for x, y in zip(a, b))


def test_learning_rate_schedule_against_the_oracle():
    tw = Twin(61)
    M = tw.M
    ref = [oracle.TensorState(M.view(M.p, i).cpu().numpy(), oracle.E4M3, oracle.E5M2) for i in range(len(SIZES))]

    def oracle_step(t, lr):
        for i, r in enumerate(ref):
            r.step(bf16_host_bits(M.view(M.g, i)), lr, HP["beta1"], HP["beta2"], HP["eps"], HP["weight_decay"], t)

    tw.grads(1)
    tw.opt.step()  # step 1 (the amax pre-pass) the regular way
    oracle_step(1, HP["lr"])
    tw.opt.set_schedule(LRS)  # steps 2 .. 7
    assert tw.opt.scheduled_step() == 2
    for k, lr in enumerate(LRS):
        tw.grads(k + 2)
        tw.opt.step_scheduled()
        oracle_step(k + 2, lr)
    tw.opt.check()
    assert tw.opt.scheduled_step() == 2 + len(LRS)
    torch.cuda.synchronize()
    for i, r in enumerate(ref):
        assert (M.view(M.m, i).cpu().numpy() == r.m).all() and (M.view(M.v, i).cpu().numpy() == r.v).all(), i
        assert (M.view(M.p, i).cpu().numpy().view(np.uint32) == r.p.view(np.uint32)).all(), i
        assert float(M.scale_m[i]) == float(r.scale_m[0]) and float(M.amax_v[i]) == float(r.amax_v[0]), i


@pytest.mark.parametrize("opts", [{}, dict(stochastic_rounding=True, seed=5, amax_history_len=4, margin_v=1),
                                  dict(stochastic_rounding=True, sr_draw_bits=16, seed=5, amax_history_len=4),
                                  dict(tma=False), dict(tma=False, stochastic_rounding=True, seed=5, amax_history_len=4)],
                         ids=["default", "sr_history_margin", "sr16_history", "vector", "vector_sr_history"])
def test_captured_graph_replays_equal_regular_steps(opts):
    """One fp8adam_step_scheduled captured in a CUDA graph, replayed once per
    step with new gradients written between replays, against fp8adam_step_ex
    with the same per-step parameters (loss scale and clipping in the later
    steps)."""
    a, b = Twin(62, **opts), Twin(62, **opts)
    for tw in (a, b):
        tw.grads(1)
        tw.opt.step()
    kw = [dict(loss_scale=1.0, max_norm=0.0)] * 3 + [dict(loss_scale=256.0, max_norm=0.5)] * 3
    steps = [capi.fp8adam_step_params(lr, HP["beta1"], HP["beta2"], HP["eps"], HP["weight_decay"], k + 2,
                                      kw[k]["loss_scale"], kw[k]["max_norm"], 0) for k, lr in enumerate(LRS)]
    s = torch.cuda.current_stream()
    capi.fp8adam_set_schedule(b.opt.ctx, steps, s.cuda_stream)
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(s)
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            b.opt.step_scheduled(stream=side)  # the binding's call, device guard included
    s.wait_stream(side)
    torch.cuda.synchronize()
    assert b.opt.scheduled_step() == 2  # capture ran nothing
    for k, lr in enumerate(LRS):
        a.grads(k + 2)
        a.opt.t = k + 1
        a.opt.step(lr=lr, **kw[k])
        b.grads(k + 2)
        graph.replay()
        torch.cuda.synchronize()
        assert _same(a.state(), b.state()), k
    b.opt.check()
    assert b.opt.scheduled_step() == 2 + len(LRS)
    del graph


def test_current_scaling_schedule_from_step_1():
    a, b = Twin(63, jit_every_step=True), Twin(63, jit_every_step=True)
    b.opt.set_schedule(LRS[:4], first_step=1)
    for k, lr in enumerate(LRS[:4]):
        a.grads(k + 1)
        a.opt.step(lr=lr)
        b.grads(k + 1)
        b.opt.step_scheduled()
    assert _same(a.state(), b.state())


def test_past_the_end_updates_nothing_and_reports():
    tw = Twin(64)
    tw.grads(1)
    tw.opt.step()
    with pytest.raises(capi.Fp8AdamError):
        tw.opt.set_schedule(LRS[:2], first_step=1)  # step 1 needs the host-decided pre-pass
    tw.opt.set_schedule(LRS[:2])
    for t in (2, 3):
        tw.grads(t)
        tw.opt.step_scheduled()
    tw.opt.check()
    before = tw.state()
    tw.grads(4)
    tw.opt.step_scheduled()  # no entry for step 4
    with pytest.raises(capi.Fp8AdamError) as e:
        tw.opt.check()
    assert e.value.code == capi.ERR_SCHEDULE_END
    assert _same(before, tw.state())
    tw.opt.check()  # cleared
    tw.opt.set_schedule(LRS[:1], first_step=4)  # the schedule continues
    tw.opt.step_scheduled()
    tw.opt.check()
    assert tw.opt.scheduled_step() == 5
