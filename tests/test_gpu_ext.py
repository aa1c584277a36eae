"""The step's options through the C ABI (fp8adam_create_ex / fp8adam_step_ex)
against the oracle's extended step, free-running from the same seeded state
on the same seeded gradients.  Covered options:
- scale margin and amax history;
- update from stored moments;
- stochastic rounding, with 32-bit draws (integer encoder) and with 16-bit
  draws (the hardware stochastic-rounding conversion);
- loss-scale removal, global-norm clipping and skip-on-non-finite;
- the bf16 param copy."""
import math

import numpy as np
import pytest
import torch

import oracle
import pins
from fp8_quantized_adam_b200 import FP8AdamW, capi, workloads
from gpu_harness import HP, bf16_host_bits

pytestmark = pytest.mark.gpu

SIZES = [70001, 4096, 33, 0, 3 * 4096 + 5, 200003]


class ExtRun:
    def __init__(self, cfg, sizes=SIZES, mf=oracle.E4M3, vf=oracle.E5M2, bf16=False, specs=None, subset=None,
                 **opt):
        self.specs = specs if specs is not None else workloads.custom_layout(sizes)
        dev = torch.device("cuda:0")
        self.M = workloads.FlatModel(self.specs, dev, m_fp32=mf == oracle.FP32, v_fp32=vf == oracle.FP32)
        M = self.M
        workloads.init_params_into(self.specs, M.views(M.p), cfg)
        self.cfg = cfg
        self.sig = workloads.tensor_sigmas(self.specs, cfg)
        self.bf16 = [torch.zeros(s.numel, dtype=torch.bfloat16, device=dev) for s in self.specs] if bf16 else None
        self.opt_kw = opt
        self.opt = FP8AdamW(M.views(M.p), M.views(M.g), m_fmt=mf, v_fmt=vf, m=M.views(M.m), v=M.views(M.v),
                            scale_m=M.scale_m, scale_v=M.scale_v, amax_m=M.amax_m, amax_v=M.amax_v,
                            param_bf16=self.bf16, **opt)
        torch.cuda.synchronize()
        # the oracle runs the `subset` of tensors (all by default); tensors are independent
        self.subset = list(range(len(self.specs))) if subset is None else list(subset)
        self.ref = {i: oracle.TensorState(M.view(M.p, i).cpu().numpy(), mf, vf) for i in self.subset}
        self.t = 0
        self.flags = ((oracle.FLAG_UPDATE_FROM_STORED if opt.get("update_from_stored") else 0)
                      | (oracle.FLAG_STOCHASTIC if opt.get("stochastic_rounding") else 0)
                      | (oracle.FLAG_SR_DRAW16 if opt.get("sr_draw_bits") == 16 else 0))

    def step(self, loss_scale=1.0, max_norm=0.0, skip_nonfinite=False, poison=None, fill=None):
        self.t += 1
        M = self.M
        workloads.grads_into(self.specs, M.views(M.g), self.cfg, self.t, self.sig)
        if fill is not None:  # tensor index -> a constant gradient value
            for i, f in fill.items():
                M.view(M.g, i).fill_(f)
        if poison is not None:
            M.g[poison] = float("inf")
        self.opt.step(loss_scale=loss_scale, max_norm=max_norm, skip_nonfinite=skip_nonfinite)
        need_all = loss_scale != 1.0 or max_norm > 0 or skip_nonfinite  # the global norm
        grads = {i: bf16_host_bits(M.view(M.g, i)) for i in (range(len(self.specs)) if need_all else self.subset)}
        gm, skip, norm = 1.0, False, None
        if loss_scale != 1.0 or max_norm > 0 or skip_nonfinite:
            sumsq, bad = oracle.grad_sumsq([grads[i] for i in range(len(self.specs))])
            gm = oracle.grad_multiplier(sumsq, loss_scale, max_norm)
            skip = bool(skip_nonfinite and bad > 0)
            norm = math.sqrt(sumsq) / loss_scale
        for i, r in self.ref.items():
            r.step_ex(grads[i], HP["lr"], HP["beta1"], HP["beta2"], HP["eps"], HP["weight_decay"], self.t,
                      self.flags, margin_m=self.opt_kw.get("margin_m", 0), margin_v=self.opt_kw.get("margin_v", 0),
                      hist_len=self.opt_kw.get("amax_history_len", 0), seed=self.opt_kw.get("seed", 0),
                      tensor_index=self.opt_kw.get("sr_tensor_ids", range(len(self.specs)))[i], grad_mult=gm,
                      skip=skip, want_bf16=self.bf16 is not None)
        return norm, skip

    def compare(self):
        torch.cuda.synchronize()
        M = self.M
        for i, r in self.ref.items():
            for name, got, exp in (("p", M.view(M.p, i), r.p), ("m", M.view(M.m, i), r.m), ("v", M.view(M.v, i), r.v)):
                g = got.cpu().numpy()
                assert (g.view(np.uint8) == exp.view(np.uint8)).all(), (i, name, np.flatnonzero(g != exp)[:5])
            for name, arr, exp in (("scale_m", M.scale_m, r.scale_m), ("scale_v", M.scale_v, r.scale_v),
                                   ("amax_m", M.amax_m, r.amax_m), ("amax_v", M.amax_v, r.amax_v)):
                assert np.float32(arr[i].item()).view(np.uint32) == exp.view(np.uint32)[0], (i, name)
            if self.bf16 is not None and r.p.size:
                b = self.bf16[i].cpu().view(torch.int16).numpy().view(np.uint16)
                assert (b == r.p_bf16).all(), (i, "bf16")
            if getattr(r, "hist_m", None) is not None:
                h = self.opt.hist_m[:, i].cpu().numpy()
                assert (h.view(np.uint32) == r.hist_m.view(np.uint32)).all(), (i, "hist_m")


@pytest.mark.parametrize("tma", [True, False], ids=["staged", "vector"])
def test_margin_and_amax_history(tma):
    r = ExtRun(41, margin_m=1, margin_v=2, amax_history_len=4, tma=tma)
    for _ in range(9):
        r.step()
        r.compare()


def test_margin_with_subnormal_amax():
    """Gradients of 1e-21 make v ~5e-44 (an fp32 subnormal): its scale with a
    large margin depends on the subnormal's exact exponent."""
    r = ExtRun(48, margin_m=20, margin_v=30)
    for _ in range(4):
        r.step(fill={1: 1e-21})
        r.compare()
    assert 0 < float(r.M.amax_v[1]) < 1.2e-38


@pytest.mark.parametrize("vf", [oracle.E5M2, oracle.E4M3], ids=["v5", "v4"])
def test_update_from_stored_moments(vf):
    r = ExtRun(42, vf=vf, update_from_stored=True)
    for _ in range(5):
        r.step()
        r.compare()


DRAWS = pytest.mark.parametrize("draws", [32, 16], ids=["d32", "d16"])


@DRAWS
@pytest.mark.parametrize("tma", [True, False], ids=["staged", "vector"])
@pytest.mark.parametrize("fmts", [(oracle.E4M3, oracle.E5M2), (oracle.E5M2, oracle.E4M3)], ids=["m4v5", "m5v4"])
def test_stochastic_rounding(fmts, tma, draws):
    """The lean staged kernel (no other option) or the per-thread kernel, on
    tensors of 0, 33 and ragged sizes among whole ones: codes, params, scales
    and amax equal the oracle's bit for bit over five steps."""
    r = ExtRun(43, mf=fmts[0], vf=fmts[1], stochastic_rounding=True, seed=0x0123456789ABCDEF, tma=tma,
               sr_draw_bits=draws)
    for _ in range(5):
        r.step()
        r.compare()


@DRAWS
def test_stochastic_rounding_with_a_loss_scale(draws):
    """Stochastic rounding with a loss scale and no clipping: the multiplier
    1/loss_scale is a kernel argument, so the staged kernel that keeps the
    multiply runs (the lean one assumes multiplier 1); codes, params, scales
    and amax equal the oracle's bit for bit."""
    r = ExtRun(54, stochastic_rounding=True, seed=0xABCDEF, sr_draw_bits=draws)
    for ls in (4.0, 1000.0, 1.0, 65536.0):
        r.step(loss_scale=ls)
        r.compare()


@pytest.mark.parametrize("vf", [oracle.E5M2, oracle.E4M3], ids=["v5", "v4"])
def test_sr16_with_update_from_stored_and_bf16_copy(vf):
    """16-bit-draw stochastic rounding in the staged kernel with every option
    compiled in: the update reads the stored (stochastically rounded) codes
    and the bf16 copy is written; bit for bit against the oracle."""
    r = ExtRun(55, vf=vf, bf16=True, update_from_stored=True, stochastic_rounding=True, seed=31337,
               sr_draw_bits=16, margin_v=1)
    for _ in range(5):
        r.step()
        r.compare()


def test_sr16_draw_flag_needs_stochastic_rounding():
    dev = torch.device("cuda:0")
    p = [torch.zeros(100, device=dev)]
    g = [torch.zeros(100, device=dev, dtype=torch.bfloat16)]
    with pytest.raises(capi.Fp8AdamError) as e:
        FP8AdamW(p, g, sr_draw_bits=16)
    assert e.value.code == capi.ERR_INVALID_ARG
    with pytest.raises(ValueError):
        FP8AdamW(p, g, stochastic_rounding=True, sr_draw_bits=8)


@pytest.mark.parametrize("tma", [True, False], ids=["staged", "vector"])
def test_bf16_param_copy(tma):
    r = ExtRun(44, bf16=True, tma=tma)
    for _ in range(3):
        r.step()
        r.compare()


@pytest.mark.parametrize("tma", [True, False], ids=["staged", "vector"])
def test_loss_scale_clip_and_skip(tma):
    r = ExtRun(45, tma=tma)
    for ls, mx in ((1024.0, 1.0), (1.0, 0.05), (65536.0, 0.0), (8.0, 1e-4)):
        norm, skip = r.step(loss_scale=ls, max_norm=mx, skip_nonfinite=True)
        r.compare()
        gn, sk = r.opt.grad_info()
        assert sk == 0 and math.isclose(gn, norm, rel_tol=1e-12)
    # an inf gradient: the whole step is skipped on both sides
    before = r.M.p.clone()
    norm, skip = r.step(loss_scale=2.0, max_norm=1.0, skip_nonfinite=True, poison=123)
    assert skip
    r.compare()
    assert r.opt.grad_info()[1] == 1
    assert torch.equal(before, r.M.p)


@pytest.mark.parametrize("tma", [True, False], ids=["staged", "vector"])
def test_loss_scale_alone_runs_no_prepass(tma):
    """A loss scale without clipping or skipping (as ZeRO-1's 1/world
    average): the multiplier 1/loss_scale is a kernel argument, so no
    grad-norm pre-pass runs (one launch per step after step 1's amax
    pre-pass), and the results equal the oracle's with the pinned multiplier,
    for power-of-two scales and others."""
    r = ExtRun(48, tma=tma)
    for t, ls in enumerate((1024.0, 3.0, 65536.0, 1000.0), start=1):
        before = capi.fp8adam_launch_count()
        r.step(loss_scale=ls)
        assert capi.fp8adam_launch_count() - before == (2 if t == 1 else 1), t
        r.compare()


def test_prepass_only_equals_default_kernel():
    """skip_nonfinite alone (multiplier 1, nothing skipped) runs the variant
    kernels; the results equal the default step bit for bit."""
    a = ExtRun(46)
    b = ExtRun(46)
    for _ in range(3):
        a.step(skip_nonfinite=True)
        b.step()
    torch.cuda.synchronize()
    for x in ("p", "m", "v", "scale_m", "scale_v", "amax_m", "amax_v"):
        assert torch.equal(getattr(a.M, x).view(torch.uint8), getattr(b.M, x).view(torch.uint8)), x


@DRAWS
def test_options_with_fp32_moments_and_current_scaling(draws):
    """One fp32 moment (per-thread kernel) and current scaling (an amax
    pre-pass every step), with a margin, stochastic rounding, a loss scale and
    clipping."""
    r = ExtRun(47, mf=oracle.FP32, vf=oracle.E5M2, margin_v=1, stochastic_rounding=True, seed=5,
               jit_every_step=True, sr_draw_bits=draws)
    r.flags |= oracle.FLAG_JIT_EVERY_STEP
    for _ in range(4):
        r.step(loss_scale=4.0, max_norm=0.5)
        r.compare()


@DRAWS
def test_options_on_misaligned_views(draws):
    """Buffers (and the bf16 outputs) that start one element into their
    allocation take the element-by-element path of the staged variant
    kernel; stochastic rounding, a margin, the history and the bf16 copy must
    still match the oracle bit for bit."""
    dev = torch.device("cuda:0")
    ns = [33, 4097, 70000]
    p = [torch.zeros(n + 1, device=dev)[1:] for n in ns]
    g = [torch.zeros(n + 1, device=dev, dtype=torch.bfloat16)[1:] for n in ns]
    m = [torch.zeros(n + 1, device=dev, dtype=torch.uint8)[1:] for n in ns]
    v = [torch.zeros(n + 1, device=dev, dtype=torch.uint8)[1:] for n in ns]
    pb = [torch.zeros(n + 1, device=dev, dtype=torch.bfloat16)[1:] for n in ns]
    specs = workloads.custom_layout(ns)
    workloads.init_params_into(specs, p, 49)
    kw = dict(stochastic_rounding=True, seed=99, margin_m=1, amax_history_len=3, sr_draw_bits=draws)
    opt = FP8AdamW(p, g, m=m, v=v, param_bf16=pb, **kw)
    ref = [oracle.TensorState(x.cpu().numpy(), oracle.E4M3, oracle.E5M2) for x in p]
    sig = workloads.tensor_sigmas(specs, 49)
    flags = oracle.FLAG_STOCHASTIC | (oracle.FLAG_SR_DRAW16 if draws == 16 else 0)
    for t in range(1, 5):
        workloads.grads_into(specs, g, 49, t, sig)
        opt.step(loss_scale=2.0)
        grads = [bf16_host_bits(x) for x in g]
        sumsq, _ = oracle.grad_sumsq(grads)
        gm = oracle.grad_multiplier(sumsq, 2.0, 0.0)
        for i, rs in enumerate(ref):
            rs.step_ex(grads[i], HP["lr"], HP["beta1"], HP["beta2"], HP["eps"], HP["weight_decay"], t, flags,
                       margin_m=1, hist_len=3, seed=99, tensor_index=i, grad_mult=gm, want_bf16=True)
    torch.cuda.synchronize()
    for i, rs in enumerate(ref):
        assert (m[i].cpu().numpy() == rs.m).all() and (v[i].cpu().numpy() == rs.v).all(), i
        assert (p[i].cpu().numpy().view(np.uint32) == rs.p.view(np.uint32)).all(), i
        assert (pb[i].cpu().view(torch.int16).numpy().view(np.uint16) == rs.p_bf16).all(), i


@DRAWS
def test_options_through_host_step(draws):
    """fp8adam_step_host with options: the history and stochastic rounding
    (grouped steps), then loss scale and clipping (one group after all
    copies); the same results as copying the gradients and fp8adam_step_ex."""
    a = ExtRun(50, amax_history_len=3, stochastic_rounding=True, seed=7, sr_draw_bits=draws)
    b = ExtRun(50, amax_history_len=3, stochastic_rounding=True, seed=7, sr_draw_bits=draws)
    h = torch.empty(b.M.g.numel(), dtype=torch.bfloat16, pin_memory=True)
    views = [h[o:o + s.numel] for o, s in zip(b.M.off, b.specs)]
    for t in range(1, 6):
        kw = dict(loss_scale=64.0, max_norm=0.5) if t >= 4 else {}
        a.step(**kw)
        workloads.grads_into(b.specs, b.M.views(b.M.g), b.cfg, t, b.sig)
        h.copy_(b.M.g)
        b.M.g.zero_()
        b.opt.step_host(views, **kw)
        torch.cuda.synchronize()
        for x in ("p", "m", "v", "scale_m", "scale_v", "amax_m", "amax_v"):
            assert torch.equal(getattr(a.M, x).view(torch.uint8), getattr(b.M, x).view(torch.uint8)), (t, x)
        assert torch.equal(a.opt.hist_m, b.opt.hist_m)
    a.compare()  # and a against the oracle


@DRAWS
def test_options_on_the_llama2_100m_layout(draws):
    """Stochastic rounding, a 16-step history, margins and the bf16 copy on
    the 110-tensor Llama2-100M layout in the launch configuration the bench
    times (guided chunk table, staged kernel); the embedding, the first and
    last layer's matrices and a norm gain against the oracle, bit for bit."""
    specs = workloads.layout("llama2_100m")
    subset = [0, 1, 5, len(specs) - 2, len(specs) - 1]
    r = ExtRun(52, specs=specs, subset=subset, bf16=True, stochastic_rounding=True, seed=77,
               amax_history_len=16, margin_m=1, margin_v=2, sr_draw_bits=draws)
    for _ in range(3):
        r.step()
    r.compare()


@DRAWS
def test_lean_stochastic_rounding_on_the_llama2_100m_layout(draws):
    """The lean stochastic-rounding kernels (no other option) on the
    Llama2-100M layout in the bench's launch configuration: the guided chunk
    table, the staged kernel; a subset of tensors against the oracle."""
    specs = workloads.layout("llama2_100m")
    subset = [0, 2, 7, len(specs) - 1]
    r = ExtRun(56, specs=specs, subset=subset, stochastic_rounding=True, seed=2024, sr_draw_bits=draws)
    for _ in range(3):
        r.step()
    r.compare()


@pytest.mark.slow
@DRAWS
def test_stochastic_rounding_60_steps_on_the_llama2_100m_layout(draws):
    """Free-running stochastic rounding (lean kernels) over 60 steps of the
    Llama2-100M layout: two projections, an FFN matrix and a norm gain against
    the oracle, bit for bit, at steps 1, 20, 40 and 60 (the embedding is in
    the shorter layout tests)."""
    specs = workloads.layout("llama2_100m")
    subset = [3, 6, 7, len(specs) - 2]
    r = ExtRun(57, specs=specs, subset=subset, stochastic_rounding=True, seed=0xFEED, sr_draw_bits=draws)
    for t in range(1, 61):
        r.step()
        if t in (1, 20, 40, 60):
            r.compare()
    r.opt.check()


@pytest.mark.slow
def test_stochastic_rounding_counter_beyond_2_pow_33():
    """One tensor of 2^33 + 2*4096 + 5 elements, stochastic rounding on,
    inputs periodic in 4096 elements, step 1 from the zero state.  Element j's
    random words are Philox4x32-10 of counter (j/2 low, j/2 high, tensor,
    step): past element 2^33 the counter's high word changes, and the chunk
    table is cut there.  The codes of sampled elements on both sides of 2^33
    and at the end must equal the oracle's SR encoder fed with the oracle's
    Philox bits for those very indices; the params (which do not depend on the
    rounding) equal the oracle's step on one period, bit for bit."""
    period = 4096
    n = (1 << 33) + 2 * period + 5
    seed = 0x5EED0FF1CE
    dev = torch.device("cuda:0")
    base = workloads.custom_layout([period])
    pp = torch.zeros(period)
    workloads.init_params_into(base, [pp], 53)
    gg = torch.zeros(period, dtype=torch.bfloat16)
    workloads.grads_into(base, [gg], 53, 1, workloads.tensor_sigmas(base, 53))
    reps = (n + period - 1) // period
    p = pp.to(dev).repeat(reps)[:n]
    g = gg.to(dev).repeat(reps)[:n]
    m = torch.zeros(n, dtype=torch.uint8, device=dev)
    v = torch.zeros(n, dtype=torch.uint8, device=dev)
    opt = FP8AdamW([p], [g], m=[m], v=[v], stochastic_rounding=True, seed=seed)
    opt.step()
    opt.check()
    # the oracle on one period: the scales (from the step-1 amax, equal for
    # the periodic tensor) and the params
    ref = oracle.TensorState(pp.numpy(), oracle.E4M3, oracle.E5M2)
    gbits = bf16_host_bits(gg)
    ref.step_ex(gbits, HP["lr"], HP["beta1"], HP["beta2"], HP["eps"], HP["weight_decay"], 1,
                oracle.FLAG_STOCHASTIC, seed=seed, tensor_index=0)
    assert float(opt.scale_m[0]) == float(ref.scale_m[0]) and float(opt.scale_v[0]) == float(ref.scale_v[0])
    assert float(opt.amax_m[0]) == float(ref.amax_m[0]) and float(opt.amax_v[0]) == float(ref.amax_v[0])
    # step 1 from zero moments: m = 0 + (1 - b1) g and v = 0 + (1 - b2) g^2, one
    # fp32 rounding each, as the oracle's op order has them
    c = oracle.step_constants(HP["lr"], HP["beta1"], HP["beta2"], HP["eps"], HP["weight_decay"], 1)
    omb1, omb2 = np.float32(c[1]), np.float32(c[3])
    gf = pins.bf16_bits_to_f32(gbits)
    s_m, s_v = np.float32(ref.scale_m[0]), np.float32(ref.scale_v[0])
    two33 = 1 << 33
    starts = [two33 - 3 * period - 64, two33 - 64, two33 + period - 64, n - 200]  # all inside [0, n - 192]
    assert all(0 <= st and st + 192 <= n for st in starts)
    for st in starts:
        k = 192
        got_m = m[st:st + k].cpu().numpy()
        got_v = v[st:st + k].cpu().numpy()
        got_p = p[st:st + k].cpu().numpy()
        for o in range(k):
            j = st + o
            gj = gf[j % period]
            xm = np.float32(np.float32(omb1 * gj) * s_m)
            xv = np.float32(np.float32(omb2 * np.float32(gj * gj)) * s_v)
            em = oracle.encode_sr(oracle.E4M3, float(xm), oracle.sr_bits(seed, 0, 1, j, 0))
            ev = oracle.encode_sr(oracle.E5M2, float(xv), oracle.sr_bits(seed, 0, 1, j, 1))
            assert got_m[o] == em and got_v[o] == ev, (j, got_m[o], em, got_v[o], ev)
        assert (got_p.view(np.uint32) == ref.p[(np.arange(st, st + k) % period)].view(np.uint32)).all()
    opt.close()
    # the same step with 16-bit draws on the same buffers (reset in place):
    # element j's word comes from the call of j/8, whose counter passes 2^30
    # past element 2^33, and the staged kernel's element indices pass 2^32
    full = n // period
    p[:full * period].view(full, period).copy_(pp.to(dev).unsqueeze(0).expand(full, period))
    p[full * period:].copy_(pp[:n - full * period].to(dev))
    m.zero_()
    v.zero_()
    opt = FP8AdamW([p], [g], m=[m], v=[v], stochastic_rounding=True, sr_draw_bits=16, seed=seed)
    opt.step()
    opt.check()
    assert float(opt.scale_m[0]) == float(ref.scale_m[0]) and float(opt.scale_v[0]) == float(ref.scale_v[0])
    for st in starts:
        k = 192
        got_m = m[st:st + k].cpu().numpy()
        got_v = v[st:st + k].cpu().numpy()
        got_p = p[st:st + k].cpu().numpy()
        for o in range(k):
            j = st + o
            gj = gf[j % period]
            xm = np.float32(np.float32(omb1 * gj) * s_m)
            xv = np.float32(np.float32(omb2 * np.float32(gj * gj)) * s_v)
            em = oracle.encode_sr16(oracle.E4M3, float(xm), oracle.sr16_bits(seed, 0, 1, j, 0))
            ev = oracle.encode_sr16(oracle.E5M2, float(xv), oracle.sr16_bits(seed, 0, 1, j, 1))
            assert got_m[o] == em and got_v[o] == ev, (j, got_m[o], em, got_v[o], ev)
        assert (got_p.view(np.uint32) == ref.p[(np.arange(st, st + k) % period)].view(np.uint32)).all()
    opt.close()


@DRAWS
def test_stochastic_rounding_does_not_depend_on_the_chunk_table(draws):
    """Each element's draw is a function of its index, tensor and step alone,
    so chunk lengths of 4K, 64K and 128K elements and the guided table (and
    with them the staged kernel's pairing of threads) give the same codes and
    params, bit for bit, over four steps."""
    outs = []
    for chunk in (4096, 65536, 131072, 0):
        r = ExtRun(58, sizes=[70001, 4096, 33, 3 * 65536 + 4099, 200003], stochastic_rounding=True, seed=11,
                   sr_draw_bits=draws, chunk_elems=chunk, subset=[])
        for _ in range(4):
            r.step()
        torch.cuda.synchronize()
        outs.append([x.clone() for x in (r.M.p, r.M.m, r.M.v, r.M.scale_m, r.M.scale_v, r.M.amax_m, r.M.amax_v)])
        r.opt.check()
        r.opt.close()
    for o in outs[1:]:
        for a, b in zip(outs[0], o):
            assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))


@DRAWS
def test_sr_tensor_ids_key_the_draws(draws):
    """Caller-given counter words (sr_tensor_ids): tensor i draws as the
    oracle's tensor ids[i] (here large, out of order, and one shared), bit for
    bit, over three steps; without them the codes differ."""
    ids = [7, 1 << 31, 3, 99, 3, 0xFFFFFFFF]
    r = ExtRun(59, stochastic_rounding=True, seed=4242, sr_draw_bits=draws, sr_tensor_ids=ids)
    plain = ExtRun(59, stochastic_rounding=True, seed=4242, sr_draw_bits=draws, subset=[])
    for _ in range(3):
        r.step()
        plain.step()
        r.compare()
    torch.cuda.synchronize()
    assert not torch.equal(r.M.m, plain.M.m)


@DRAWS
def test_checkpoint_resume_with_stochastic_rounding_is_bitwise(draws):
    """Ten SR steps in one go equal five, a checkpoint, a fresh optimizer on
    fresh buffers restored from it, and five more, bit for bit: the step
    index, seed, draw width and tensor ids carry the random stream.  A
    checkpoint refuses to load into an optimizer with another seed."""
    kw = dict(stochastic_rounding=True, seed=777, sr_draw_bits=draws, subset=[])
    a = ExtRun(60, **kw)
    for _ in range(10):
        a.step()
    b = ExtRun(60, **kw)
    for _ in range(5):
        b.step()
    sd = b.opt.state_dict()
    c = ExtRun(60, **kw)
    c.opt.load_state_dict(sd)
    c.t = b.t
    for _ in range(5):
        c.step()
    torch.cuda.synchronize()
    for x in ("p", "m", "v", "scale_m", "scale_v", "amax_m", "amax_v"):
        assert torch.equal(getattr(a.M, x).view(torch.uint8), getattr(c.M, x).view(torch.uint8)), x
    other = ExtRun(60, stochastic_rounding=True, seed=778, sr_draw_bits=draws, subset=[])
    with pytest.raises(ValueError):
        other.opt.load_state_dict(sd)


@pytest.mark.parametrize("fmts", [(oracle.E4M3, oracle.E4M3), (oracle.E5M2, oracle.E5M2)], ids=["m4v4", "m5v5"])
@pytest.mark.parametrize("tma", [True, False], ids=["staged", "vector"])
def test_sr16_same_format_pairs_with_current_scaling(fmts, tma):
    """16-bit-draw stochastic rounding for the pairs with one format for both
    moments (the staged kernel's E4M3/E4M3 and E5M2/E5M2 instances, or the
    per-thread kernel), with current scaling: bit for bit over four steps."""
    r = ExtRun(61, mf=fmts[0], vf=fmts[1], stochastic_rounding=True, seed=99, sr_draw_bits=16, tma=tma,
               jit_every_step=True)
    r.flags |= oracle.FLAG_JIT_EVERY_STEP
    for _ in range(4):
        r.step()
        r.compare()
