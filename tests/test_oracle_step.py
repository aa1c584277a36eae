"""Pins of the oracle's AdamW step (CPU).

Each test checks the oracle against something other than itself: closed
forms of the update, ``torch.optim.AdamW`` (a library routine; the pages'
only concrete optimizer call), torch's float8 casts, and brute force.
"""
import math

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st
import pytest
import torch

import pins
from pins import E4M3, E5M2, FP32, FMAX, f32

HP = dict(lr=3e-4, beta1=0.9, beta2=0.95, eps=1e-8, wd=0.1)


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _grad(n, seed, lo=-6.0, hi=-1.0):
    rng = np.random.default_rng(seed)
    s = 10.0 ** rng.uniform(lo, hi, n)
    return _bf16_bits(rng.standard_normal(n) * s)


def _step(st, g, t, hp=HP, flags=0):
    st.step(g, hp["lr"], hp["beta1"], hp["beta2"], hp["eps"], hp["wd"], t, flags)


# ---------------------------------------------------------------- scale
def test_pow2scale_matches_bruteforce(orc):
    rng = np.random.default_rng(1)
    vals = list(10.0 ** rng.uniform(-44, 38, 4000)) + [
        2.0 ** -149, 1e-45, 2.0 ** -126, 1.75, 1.7500001, 448.0, 449.0, 57344.0, 3.4e38,
        0.0, -1.0, math.inf, math.nan, 1.0, 2.0, 0.875]
    for fmt in (E4M3, E5M2):
        for a in vals:
            a32 = f32(a)
            got = orc.pow2scale(fmt, a32, 0.5)
            exp = pins.pow2scale_bruteforce(fmt, a32, 0.5)
            assert got == exp, (fmt, a32, got, exp)
            if math.isfinite(a32) and a32 > 0 and -126 < math.log2(got) < 126:
                assert FMAX[fmt] / 2 < a32 * got <= FMAX[fmt]


def test_step_constants_definition(orc):
    for t in (1, 2, 10, 1000):
        c = orc.step_constants(3e-4, 0.9, 0.95, 1e-8, 0.1, t)
        b1, b2, lr, wd = f32(0.9), f32(0.95), f32(3e-4), f32(0.1)
        exp = [b1, f32(1 - b1), b2, f32(1 - b2), f32(lr / (1 - b1 ** t)),
               f32(1 / math.sqrt(1 - b2 ** t)), f32(1e-8), f32(1 - lr * wd)]
        assert [float(x) for x in c] == exp


# ---------------------------------------------------------------- closed forms
def test_fp32_moments_constant_grad_closed_form(orc):
    """fp32 moments, m0 = v0 = 0, constant g: the bias-corrected moments are g
    and g^2 at every step, so the update is lr*g/(|g|+eps) after decay."""
    n = 4096
    rng = np.random.default_rng(3)
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    g = _grad(n, 4)
    gf = pins.bf16_bits_to_f32(g).astype(np.float64)
    st = orc.TensorState(p0, FP32, FP32)
    p_prev = p0.astype(np.float64)
    lr, wd, eps = f32(HP["lr"]), f32(HP["wd"]), f32(HP["eps"])
    for t in range(1, 51):
        _step(st, g, t)
        exp = p_prev * (1 - lr * wd) - lr * gf / (np.abs(gf) + eps)
        # moments accumulate ~t rounding errors of 2^-24
        assert np.allclose(st.p, exp, rtol=2e-6, atol=lr * 1e-5)
        mhat = st.m.astype(np.float64) / (1 - f32(HP["beta1"]) ** t)
        vhat = st.v.astype(np.float64) / (1 - f32(HP["beta2"]) ** t)
        assert np.allclose(mhat, gf, rtol=1e-5, atol=0)
        assert np.allclose(vhat, gf * gf, rtol=1e-5, atol=0)
        p_prev = st.p.astype(np.float64)


@pytest.mark.parametrize("fmts", [(E4M3, E5M2), (E4M3, E4M3), (E5M2, E5M2), (E5M2, E4M3)])
def test_zero_betas_reduce_to_codec_and_sign_sgd(orc, fmts):
    """beta1 = beta2 = 0, wd = 0: m = g, v = g^2 (exact for bf16 g), codes are
    the float8 encodings of g*s, and the step is p - lr*g/(|g| + eps)."""
    mf, vf = fmts
    n = 3000
    rng = np.random.default_rng(5)
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    hp = dict(lr=1e-3, beta1=0.0, beta2=0.0, eps=1e-8, wd=0.0)
    st = orc.TensorState(p0, mf, vf)
    for t in (1, 2, 3):
        g = _grad(n, 10 + t, -4, 0)
        gf = pins.bf16_bits_to_f32(g)
        prev_am, prev_av, sm, sv = float(st.amax_m[0]), float(st.amax_v[0]), float(st.scale_m[0]), float(st.scale_v[0])
        p_before = st.p.astype(np.float64)
        _step(st, g, t, hp)
        gg = gf.astype(np.float64) ** 2  # exact in fp32 too (bf16 has 8 bits)
        am, av = float(np.abs(gf).max()), float(gg.max())
        assert float(st.amax_m[0]) == am and float(st.amax_v[0]) == av
        s_m = pins.pow2scale_bruteforce(mf, am if t == 1 else prev_am, sm)
        s_v = pins.pow2scale_bruteforce(vf, av if t == 1 else prev_av, sv)
        assert float(st.scale_m[0]) == s_m and float(st.scale_v[0]) == s_v
        xm = torch.from_numpy(gf.astype(np.float64) * s_m).float().clamp(-FMAX[mf], FMAX[mf])
        xv = torch.from_numpy(gg * s_v).float().clamp(-FMAX[vf], FMAX[vf])
        assert (st.m == pins.torch_encode(mf, xm).numpy()).all()
        assert (st.v == pins.torch_encode(vf, xv).numpy()).all()
        exp = p_before - f32(1e-3) * gf / (np.abs(gf) + f32(1e-8))
        assert np.allclose(st.p, exp, rtol=1e-6, atol=1e-9)


def test_first_step_quantises_exact_moments_without_saturation(orc):
    """Step 1 from zero state: m = (1-b1)*g and v = (1-b2)*g^2 exactly as fp32
    products; the step-1 scale comes from this step's own amax, so nothing
    saturates and amax*scale lies in (max/2, max]."""
    n = 1 << 14
    g = _grad(n, 21)
    gf = pins.bf16_bits_to_f32(g)
    st = orc.TensorState(np.zeros(n, np.float32), E4M3, E5M2)
    _step(st, g, 1)
    omb1, omb2 = np.float32(f32(1 - f32(0.9))), np.float32(f32(1 - f32(0.95)))
    m = omb1 * gf
    v = omb2 * (gf * gf)
    assert float(st.amax_m[0]) == float(np.abs(m).max())
    assert float(st.amax_v[0]) == float(v.max())
    sm, sv = float(st.scale_m[0]), float(st.scale_v[0])
    assert FMAX[E4M3] / 2 < float(st.amax_m[0]) * sm <= FMAX[E4M3]
    assert FMAX[E5M2] / 2 < float(st.amax_v[0]) * sv <= FMAX[E5M2]
    assert (st.m == pins.torch_encode(E4M3, torch.from_numpy(m * np.float32(sm))).numpy()).all()
    assert (st.v == pins.torch_encode(E5M2, torch.from_numpy(v * np.float32(sv))).numpy()).all()
    assert int(st.stats[1]) == 0


def test_weight_decay_only(orc):
    """g = 0: the moments stay 0 and p is only decayed by (1 - lr*wd)."""
    n = 777
    rng = np.random.default_rng(8)
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    st = orc.TensorState(p0, E4M3, E5M2)
    g = np.zeros(n, np.uint16)
    p = p0.copy()
    for t in range(1, 6):
        _step(st, g, t)
        p = p * np.float32(f32(1 - f32(HP["lr"]) * f32(HP["wd"])))
        assert (st.p.view(np.uint32) == p.view(np.uint32)).all()
        assert (st.m == 0).all() and (st.v == 0).all()
        assert float(st.amax_m[0]) == 0.0 and float(st.scale_m[0]) == 1.0  # scale kept


# ---------------------------------------------------------------- library pins
def test_fp32_moments_match_torch_adamw(orc):
    """fp32 moments against torch.optim.AdamW (foreach=False): 10 steps
    free-running on params (rel 1e-6), and per step, starting torch from the
    oracle's state, m and v within a few ulps of their addends."""
    n = 1 << 13
    rng = np.random.default_rng(11)
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    st = orc.TensorState(p0, FP32, FP32)
    free = pins.TorchFakeQuantAdamW(p0, FP32, FP32, **HP)
    for t in range(1, 11):
        g = _grad(n, 100 + t)
        forced = pins.TorchFakeQuantAdamW(st.p, FP32, FP32, **HP)
        forced.mq, forced.vq = torch.from_numpy(st.m.copy()), torch.from_numpy(st.v.copy())
        forced.t = t - 1
        m_prev, v_prev = st.m.astype(np.float64), st.v.astype(np.float64)
        _step(st, g, t)
        forced.step(g)
        free.step(g)
        assert pins.params_close(st.p, free.p, HP["lr"], t)
        assert pins.params_close(st.p, forced.p, HP["lr"], 1)
        # m = b1*m + (1-b1)*g may cancel: bound by a few ulps of the addends
        gf = pins.bf16_bits_to_f32(g).astype(np.float64)
        bound_m = 2.0 ** -21 * (0.9 * np.abs(m_prev) + 0.1 * np.abs(gf))
        bound_v = 2.0 ** -21 * (0.95 * v_prev + 0.05 * gf * gf)
        assert (np.abs(st.m - forced.m_unq.numpy()) <= bound_m).all()
        assert (np.abs(st.v - forced.v_unq.numpy()) <= bound_v).all()


def _codes_within_rounding(orc, fmt, q, x, delta):
    """True where code q is the encoding of some value in [x - delta,
    x + delta] (torch's own float8 cast of the two ends brackets it)."""
    lo = pins.torch_encode(fmt, torch.from_numpy(np.clip(x - delta, -FMAX[fmt], FMAX[fmt]).astype(np.float32)))
    hi = pins.torch_encode(fmt, torch.from_numpy(np.clip(x + delta, -FMAX[fmt], FMAX[fmt]).astype(np.float32)))
    v, vlo, vhi = orc.decode(fmt, q), orc.decode(fmt, lo.numpy()), orc.decode(fmt, hi.numpy())
    return (np.minimum(vlo, vhi) <= v) & (v <= np.maximum(vlo, vhi))


def _teacher_forced_compare(orc, mf, vf, n, steps, seed, jit=False):
    """At every step, torch's AdamW with float8-stored moments starts from the
    oracle's own state.  torch orders the fp32 operations differently (e.g.
    m.lerp_(g, 1-b1)), so its m, v differ from the oracle's by a few ulps of
    the EMA's addends.  A code may differ only where such a perturbation of
    torch's value reaches the oracle's code (values at a rounding midpoint, or
    m cancelling to a tiny value); params agree to 1e-6 of the update."""
    rng = np.random.default_rng(seed)
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    st = orc.TensorState(p0, mf, vf)
    flips = 0
    for t in range(1, steps + 1):
        g = _grad(n, seed * 1000 + t)
        gf = np.abs(pins.bf16_bits_to_f32(g).astype(np.float64))
        p_before = st.p.copy()
        m_old = np.abs(orc.decode(mf, st.m).astype(np.float64)) / float(st.scale_m[0])
        v_old = np.abs(orc.decode(vf, st.v).astype(np.float64)) / float(st.scale_v[0])
        sim = pins.TorchFakeQuantAdamW(st.p, mf, vf, **HP)
        sim.mq = torch.from_numpy(st.m.copy())
        sim.vq = torch.from_numpy(st.v.copy())
        sim.scale_m, sim.scale_v = float(st.scale_m[0]), float(st.scale_v[0])
        sim.amax_m, sim.amax_v = float(st.amax_m[0]), float(st.amax_v[0])
        sim.t = t - 1
        sim.step(g, jit_every_step=jit)
        _step(st, g, t, flags=orc.FLAG_JIT_EVERY_STEP if jit else 0)
        assert float(st.scale_m[0]) == sim.scale_m and float(st.scale_v[0]) == sim.scale_v
        assert math.isclose(float(st.amax_m[0]), sim.amax_m, rel_tol=1e-6)
        assert math.isclose(float(st.amax_v[0]), sim.amax_v, rel_tol=1e-6)
        addend_m = 0.9 * m_old + 0.1 * gf
        addend_v = 0.95 * v_old + 0.05 * gf * gf
        for q, qs, fmt, unq, s, add in (
                (st.m, sim.mq.numpy(), mf, sim.m_unq.numpy(), sim.scale_m, addend_m),
                (st.v, sim.vq.numpy(), vf, sim.v_unq.numpy(), sim.scale_v, addend_v)):
            d = np.flatnonzero(q != qs)
            flips += d.size
            x = unq[d].astype(np.float64) * s
            delta = 4 * 2.0 ** -24 * add[d] * s
            assert _codes_within_rounding(orc, fmt, q[d], x, delta).all()
        assert pins.params_close(st.p, sim.p, HP["lr"], 1, p_before=p_before)
    assert flips <= max(2, int(1e-3 * n * steps))
    return st


@pytest.mark.parametrize("fmts", [(E4M3, E5M2), (E4M3, E4M3), (E5M2, E5M2), (E5M2, E4M3)],
                         ids=["m4v5", "m4v4", "m5v5", "m5v4"])
def test_fp8_moments_match_torch_adamw_with_float8_storage(orc, fmts):
    _teacher_forced_compare(orc, fmts[0], fmts[1], n=1 << 13, steps=12, seed=31)


def test_current_scaling_matches_torch(orc):
    _teacher_forced_compare(orc, E4M3, E5M2, n=1 << 12, steps=6, seed=41, jit=True)


def test_single_element_stall_trajectory(orc):
    """One element, constant g = 1e-3, 300 steps, free-running against the
    torch AdamW + float8 simulation.  With round-to-nearest storage and
    delayed scaling the stored m stops moving: its code becomes constant and
    the bias-corrected m settles below g (the EMA stalls), while the update
    keeps the sign of g."""
    g = _bf16_bits(np.array([1e-3], np.float32))
    gf = float(pins.bf16_bits_to_f32(g)[0])
    st = orc.TensorState(np.zeros(1, np.float32), E4M3, E5M2)
    sim = pins.TorchFakeQuantAdamW(np.zeros(1, np.float32), E4M3, E5M2, **HP)
    codes, p_prev = [], 0.0
    for t in range(1, 301):
        _step(st, g, t)
        sim.step(g)
        assert int(st.m[0]) == int(sim.mq[0]) and int(st.v[0]) == int(sim.vq[0])
        assert float(st.scale_m[0]) == sim.scale_m and float(st.scale_v[0]) == sim.scale_v
        assert math.isclose(float(st.p[0]), float(sim.p[0]), rel_tol=1e-6, abs_tol=1e-12)
        upd = float(st.p[0]) - p_prev * f32(1 - f32(3e-4) * f32(0.1))
        assert upd < 0  # sign of -g
        p_prev = float(st.p[0])
        codes.append(int(st.m[0]))
    assert len(set(codes[50:])) == 1  # the stored m no longer moves
    mhat = orc.decode(E4M3, [codes[-1]])[0] / float(st.scale_m[0])
    assert 0.5 < mhat / gf < 0.95  # stalled below g


# ---------------------------------------------------------------- stats, edges
def test_flush_and_saturation_counters(orc):
    """flushed = v > 0 whose code is +-0; saturated = |x*s| > max."""
    n = 5000
    rng = np.random.default_rng(51)
    gf = (rng.standard_normal(n) * 10.0 ** rng.uniform(-9, -1, n)).astype(np.float32)
    g = _bf16_bits(gf)
    for vf in (E4M3, E5M2):
        st = orc.TensorState(np.zeros(n, np.float32), E4M3, vf)
        _step(st, g, 1)
        gg = pins.bf16_bits_to_f32(g)
        v = np.float32(f32(1 - f32(0.95))) * (gg * gg)
        codes = pins.torch_encode(vf, torch.from_numpy(v * np.float32(st.scale_v[0]))).numpy()
        exp_flushed = int(((v > 0) & ((codes & 0x7F) == 0)).sum())
        assert int(st.stats[0]) == exp_flushed
        assert int(st.stats[1]) == 0
    # gradients over 5 decades (v over 10): E4M3 storage of v loses far more
    # small values than E5M2
    g5 = _grad(n, 52)
    s4 = orc.TensorState(np.zeros(n, np.float32), E4M3, E4M3); _step(s4, g5, 1)
    s5 = orc.TensorState(np.zeros(n, np.float32), E4M3, E5M2); _step(s5, g5, 1)
    assert int(s4.stats[0]) > 2 * int(s5.stats[0])
    # saturation: a step-2 gradient 100x larger than step 1's overflows the
    # delayed scale
    st = orc.TensorState(np.zeros(n, np.float32), E4M3, E5M2)
    _step(st, g, 1)
    _step(st, _bf16_bits(gf * 100), 2)
    assert int(st.stats[1]) > 0


def test_empty_tensor_and_bad_arguments(orc):
    st = orc.TensorState(np.zeros(0, np.float32), E4M3, E5M2, scale_m=4.0, amax_m=3.0)
    _step(st, np.zeros(0, np.uint16), 1)
    assert float(st.scale_m[0]) == 4.0 and float(st.amax_m[0]) == 3.0
    st = orc.TensorState(np.zeros(4, np.float32), E4M3, E5M2)
    with pytest.raises(ValueError):
        _step(st, np.zeros(4, np.uint16), 0)


def test_nan_gradient_propagates_to_amax(orc):
    n = 64
    g = _grad(n, 61)
    g[5] = 0x7FC0  # bf16 NaN
    st = orc.TensorState(np.zeros(n, np.float32), E4M3, E5M2)
    _step(st, _grad(n, 60), 1)
    _step(st, g, 2)
    s_before = float(st.scale_m[0])
    assert math.isnan(float(st.amax_m[0])) and math.isnan(float(st.amax_v[0]))
    assert math.isnan(float(st.p[5])) and np.isfinite(np.delete(st.p, 5)).all()
    assert st.m[5] & 0x7F == 0x7F
    _step(st, _grad(n, 62), 3)  # a NaN amax keeps the previous scale
    assert float(st.scale_m[0]) == s_before


@settings(max_examples=30, deadline=None)
@given(lr=st.floats(1e-5, 1e-2), beta1=st.floats(0.0, 0.999), beta2=st.floats(0.5, 0.9999),
       eps=st.floats(1e-10, 1e-4), wd=st.floats(0.0, 0.3), steps=st.integers(1, 6), seed=st.integers(0, 2**31))
def test_fp32_moments_match_torch_adamw_any_hyperparameters(lr, beta1, beta2, eps, wd, steps, seed):
    """The fp32-moment step against torch.optim.AdamW for random
    hyper-parameters (a wrong bias correction, decay order or eps placement
    shows up for some beta/eps/wd), teacher-forced from the oracle's state at
    every step: params within 1e-6 of the update scale."""
    import oracle as orc

    hp = dict(lr=lr, beta1=beta1, beta2=beta2, eps=eps, wd=wd)
    n = 257
    rng = np.random.default_rng(seed)
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    s = orc.TensorState(p0, FP32, FP32)
    for t in range(1, steps + 1):
        g = _grad(n, seed + t)
        forced = pins.TorchFakeQuantAdamW(s.p, FP32, FP32, **hp)
        forced.mq, forced.vq = torch.from_numpy(s.m.copy()), torch.from_numpy(s.v.copy())
        forced.t = t - 1
        p_before = s.p.copy()
        _step(s, g, t, hp=hp)
        forced.step(g)
        assert pins.params_close(s.p, forced.p, lr, 1, p_before=p_before)
