"""Pins of the oracle's extensions (CPU).

The extensions cover several options:
- the update from the stored (requantised) moments;
- amax history and margin, as in the DelayedScaling recipe of "FP8训练的稳定性挑战…";
- stochastic rounding ("随机舍入" in its strategy list), driven by Philox4x32-10;
- the fused loss-scale / non-finite / global-norm-clip multiplier ("梯度缩放", "梯度裁剪");
- a bf16 copy of the updated params.

Each part is checked against something independent: published known-answer
vectors, statistics, closed forms, torch routines (bf16 cast, AdamW), or exact
rational arithmetic.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import pins
from pins import E4M3, E5M2, FP32, FMAX, f32

HP = dict(lr=3e-4, beta1=0.9, beta2=0.95, eps=1e-8, wd=0.1)


def _bf16_bits(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _grad(n, seed, lo=-6.0, hi=-1.0):
    rng = np.random.default_rng(seed)
    return _bf16_bits(rng.standard_normal(n) * 10.0 ** rng.uniform(lo, hi, n))


def _step(st, g, t, ex=False, flags=0, **kw):
    if ex:
        st.step_ex(g, HP["lr"], HP["beta1"], HP["beta2"], HP["eps"], HP["wd"], t, flags, **kw)
    else:
        st.step(g, HP["lr"], HP["beta1"], HP["beta2"], HP["eps"], HP["wd"], t, flags)


# ------------------------------------------------------------------ Philox
def test_philox_known_answer_vectors(orc):
    """Known-answer vectors published with Random123 (the reference
    implementation of Salmon et al., SC 2011) for philox4x32, 10 rounds."""
    kat = [
        ([0, 0, 0, 0], [0, 0], [0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8]),
        ([0xFFFFFFFF] * 4, [0xFFFFFFFF] * 2, [0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD]),
        ([0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344], [0xA4093822, 0x299F31D0],
         [0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1]),
    ]
    for ctr, key, out in kat:
        assert orc.philox4x32_10(ctr, key) == out


def test_sr_bits_are_uniform_and_distinct_per_element(orc):
    vals = np.array([orc.sr_bits(7, 3, 5, j, w) for j in range(4096) for w in (0, 1)], np.uint64)
    assert len(np.unique(vals)) == vals.size
    # top byte roughly uniform: chi-square with 255 dof well below 400
    hist = np.bincount((vals >> 24).astype(np.int64), minlength=256)
    exp = vals.size / 256
    assert ((hist - exp) ** 2 / exp).sum() < 400
    assert orc.sr_bits(7, 3, 5, 10, 0) != orc.sr_bits(7, 3, 6, 10, 0)  # differs per step
    assert orc.sr_bits(7, 3, 5, 10, 0) != orc.sr_bits(8, 3, 5, 10, 0)  # and per seed


# ------------------------------------------------------------------ SR
def _directed(fmt, x, up):
    """Round |x| toward zero (up=False) or away from zero (up=True) onto the
    format's grid, from the definition with floor/ceil in float64."""
    M = 3 if fmt == E4M3 else 2
    emin = 1 - (7 if fmt == E4M3 else 15)
    a = abs(float(x))
    if a >= FMAX[fmt]:
        return math.copysign(FMAX[fmt], x)
    e = math.frexp(a)[1] - 1 if a > 0 else emin
    q = 2.0 ** (max(e, emin) - M)
    n = math.ceil(a / q) if up else math.floor(a / q)
    return math.copysign(min(n * q, FMAX[fmt]), x)


def test_sr_extreme_draws_are_directed_rounding(orc):
    """r = 0 rounds every non-representable value away from zero; r = 2^32-1
    rounds toward zero (for (|x|-lo)/(hi-lo) <= 1 - 2^-32)."""
    rng = np.random.default_rng(5)
    xs = (rng.standard_normal(3000) * 10.0 ** rng.uniform(-9, 3, 3000)).astype(np.float32)
    for fmt in (E4M3, E5M2):
        for x in xs:
            up = orc.decode(fmt, [orc.encode_sr(fmt, float(x), 0)])[0]
            dn = orc.decode(fmt, [orc.encode_sr(fmt, float(x), 0xFFFFFFFF)])[0]
            assert up == _directed(fmt, x, True)
            assert dn == _directed(fmt, x, False)


def test_sr_is_unbiased_and_stays_on_the_two_neighbours(orc):
    rng = np.random.default_rng(6)
    for fmt in (E4M3, E5M2):
        for x in (0.3, 1.1, 37.7, 1e-3, 5e-6, -2.2, 400.0):
            x32 = f32(x)
            lo, hi = _directed(fmt, x32, False), _directed(fmt, x32, True)
            rs = rng.integers(0, 1 << 32, size=20000, dtype=np.uint64)
            vals = np.array([orc.decode(fmt, [orc.encode_sr(fmt, x32, int(r))])[0] for r in rs], np.float64)
            assert set(np.unique(vals)) <= {lo, hi}
            if lo != hi:
                pr = (abs(x32) - abs(lo)) / (abs(hi) - abs(lo))
                sd = abs(hi - lo) * math.sqrt(pr * (1 - pr) / vals.size)
                assert abs(vals.mean() - x32) <= 5 * sd + 1e-12 * abs(x32)
    # representable values, NaN, saturation
    for fmt in (E4M3, E5M2):
        for c in range(0, 0x7B):
            v = float(orc.decode(fmt, [c])[0])
            assert orc.encode_sr(fmt, v, 12345) == c
        assert orc.encode_sr(fmt, float("nan"), 0) == 0x7F
        assert orc.encode_sr(fmt, 1e9, 0) == (0x7E if fmt == E4M3 else 0x7B)


# ------------------------------------------------------------------ bf16 copy
def test_bf16_rounding_matches_torch(orc):
    rng = np.random.default_rng(9)
    hi = np.arange(1 << 16, dtype=np.uint32) << 16
    lows = np.array([0x0000, 0x7FFF, 0x8000, 0x8001, 0xFFFF, 0x4000], np.uint32)
    bits = np.concatenate([(hi[:, None] | lows[None, :]).ravel(),
                           rng.integers(0, 1 << 32, 1 << 20, dtype=np.uint64).astype(np.uint32)])
    x = bits.view(np.float32)
    ours = orc.f32_to_bf16(x)
    lib = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    nan = np.isnan(x)
    assert (ours[~nan] == lib[~nan]).all()
    assert ((ours[nan] & 0x7F80) == 0x7F80).all() and ((ours[nan] & 0x7F) != 0).all()


# ------------------------------------------------------------------ clip / unscale
def test_grad_sumsq_is_the_exact_sum(orc):
    rng = np.random.default_rng(10)
    parts = [
        _bf16_bits(rng.standard_normal(5000) * 10.0 ** rng.uniform(-30, 30, 5000)),
        _bf16_bits(np.array([1e-38, 3e-39, 1e38, -2.5, 0.0, -0.0], np.float32)),
        np.arange(0, 1 << 16, 7, dtype=np.uint32).astype(np.uint16),  # every exponent, incl. inf/nan
    ]
    s, bad = orc.grad_sumsq(parts)
    exact = Fraction(0)
    nonfinite = 0
    for p in parts:
        with np.errstate(invalid="ignore"):
            vals = pins.bf16_bits_to_f32(p).astype(np.float64)
        for v in vals:
            if not math.isfinite(v):
                nonfinite += 1
            else:
                exact += Fraction(v) ** 2
    assert bad == nonfinite
    assert s == float(exact)  # Fraction -> float rounds to nearest even


def _torch_amp_multiplier(grad_bits, loss_scale, max_norm):
    """The factor torch's mixed-precision recipe applies to the scaled
    gradients: unscale (divide by the loss scale), then
    torch.nn.utils.clip_grad_norm_(params, max_norm) -- the routine printed
    in the clip_grad_norm_ example of "FP8训练的稳定性挑战…" ("梯度裁剪") --
    all in float64.  max_norm <= 0 means no clipping (max_norm = inf for
    torch).  The factor is read back from the clipped gradients: the
    clipping coefficient is g_clipped / g_unscaled for a non-zero element,
    and the multiplier of the scaled gradients is that coefficient / S."""
    params, unscaled = [], []
    for bits in grad_bits:
        g = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).double()
        p = torch.zeros(g.numel(), dtype=torch.float64, requires_grad=True)
        p.grad = g / float(loss_scale)
        params.append(p)
        unscaled.append(p.grad.clone())
    torch.nn.utils.clip_grad_norm_(params, max_norm if max_norm > 0 else float("inf"))
    for p, u in zip(params, unscaled):
        nz = torch.nonzero(u)
        if len(nz):
            k = int(nz[0, 0])
            coef = float(p.grad[k]) / float(u[k])
            return coef / float(loss_scale), math.sqrt(sum(float((x * x).sum()) for x in unscaled))
    return 1.0 / float(loss_scale), 0.0


def _ulp32(x):
    x = abs(f32(x))
    return float(np.spacing(np.float32(x)))


def test_grad_multiplier_matches_torch_clip_grad_norm(orc):
    """The oracle's multiplier c = (1/S)*min(1, max_norm/(norm+1e-6)) with
    norm the L2 norm of the unscaled gradients, against torch's own
    unscale + clip_grad_norm_ on the same bf16 gradients: c must be torch's
    float64 factor rounded to fp32 (a tie band of 1e-9 of half an ulp
    allows for torch's own float64 rounding).  The cases cover several loss
    scales (powers of two and not), clipping off, norms on both sides of
    max_norm, max_norm within an fp32 ulp of the norm, and norms so small
    that the 1e-6 in the denominator decides the result."""
    rng = np.random.default_rng(77)
    sets = []
    for scale_exp, n_tensors in ((-3, 3), (-6, 2), (0, 4), (-9, 1)):
        sets.append([_bf16_bits(rng.standard_normal(int(rng.integers(1, 5000))) * 10.0 ** (scale_exp +
                     rng.uniform(-1, 1))) for _ in range(n_tensors)])
    cases = 0
    for grads in sets:
        sumsq, bad = orc.grad_sumsq(grads)
        assert bad == 0
        for S in (1.0, 2.0, 1024.0, 65536.0, 1000.0, 3.0):
            _, norm = _torch_amp_multiplier(grads, S, 0.0)
            maxes = [0.0, -1.0, 1.0, 0.5, 100.0, 1e-6, norm * 2.0, norm * 0.5]
            nf = f32(norm)
            maxes += [nf, float(np.nextafter(np.float32(nf), np.float32(0))),
                      float(np.nextafter(np.float32(nf), np.float32(np.inf)))]
            for mx in maxes:
                mx = f32(mx)
                c_ref, _ = _torch_amp_multiplier(grads, S, mx)
                c = orc.grad_multiplier(sumsq, S, mx)
                assert abs(c - c_ref) <= 0.5 * _ulp32(c) * (1 + 1e-9), (S, mx, norm, c, c_ref)
                cases += 1
    assert cases == 4 * 6 * 11


def test_grad_multiplier_distinguishes_plausible_mistakes(orc):
    """The torch pin above would catch each of these mistakes of the
    formula: the norm of the scaled instead of the unscaled gradients, the
    1e-6 dropped or multiplied in, and the clamp to 1 missing."""
    caught = {"scaled norm": False, "no eps": False, "eps times norm": False, "no clamp": False}
    for val, S, mx in ((1e-7, 1024.0, 1e-6), (1e-7, 1.0, 1e-6), (1e-3, 1.0, 100.0), (0.25, 4.0, 1.0)):
        grads = [_bf16_bits(np.full(100, val, np.float32))]
        sumsq, _ = orc.grad_sumsq(grads)
        c_ref, _ = _torch_amp_multiplier(grads, S, mx)
        c = orc.grad_multiplier(sumsq, S, mx)
        assert abs(c - c_ref) <= 0.5 * _ulp32(c) * (1 + 1e-9)
        norm = math.sqrt(sumsq) / S
        wrong = {
            "scaled norm": (1 / S) * min(1.0, mx / (math.sqrt(sumsq) + 1e-6)),
            "no eps": (1 / S) * min(1.0, mx / norm),
            "eps times norm": (1 / S) * min(1.0, mx / (norm * (1 + 1e-6))),
            "no clamp": (1 / S) * mx / (norm + 1e-6),
        }
        for k, w in wrong.items():
            if abs(f32(w) - c_ref) > _ulp32(c_ref):
                caught[k] = True
    assert all(caught.values()), caught


# ------------------------------------------------------------------ the extended step
@pytest.mark.parametrize("fmts", [(E4M3, E5M2), (E4M3, E4M3), (E5M2, E5M2), (E5M2, E4M3), (FP32, FP32)])
def test_ex_with_options_off_equals_the_pinned_step(orc, fmts):
    n = 5000
    rng = np.random.default_rng(11)
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    a, b = orc.TensorState(p0, *fmts), orc.TensorState(p0, *fmts)
    for t in range(1, 8):
        g = _grad(n, 200 + t)
        _step(a, g, t)
        _step(b, g, t, ex=True)
        for x in ("p", "m", "v", "scale_m", "scale_v", "amax_m", "amax_v", "stats"):
            assert (getattr(a, x).view(np.uint8) == getattr(b, x).view(np.uint8)).all(), x


def test_pow2scale_margin_matches_bruteforce(orc):
    """scale with margin = 2^(k - margin) clamped to 2^[-126, 126], k the
    largest exponent with amax * 2^k <= max (any k, also beyond the clamp)."""
    vals = [2.0 ** -149, 3 * 2.0 ** -149, 2.0 ** -140 * 1.8, 2.0 ** -127, 1e-40, 1e-30, 0.3, 448.0, 1e30]
    for fmt in (E4M3, E5M2):
        for a in vals:
            a32 = f32(a)
            k = max(kk for kk in range(-300, 400) if a32 * 2.0 ** kk <= FMAX[fmt])
            for margin in (0, 1, 5, 20, 64):
                exp = 2.0 ** min(126, max(-126, k - margin))
                assert orc.pow2scale(fmt, a32, 0.5, margin) == exp, (fmt, a32, margin)


def test_margin_and_amax_history(orc):
    """scale = largest 2^k with max(last H amax) * 2^k <= max, minus margin."""
    n, H = 3000, 4
    st = orc.TensorState(np.zeros(n, np.float32), E4M3, E5M2)
    hist_m, hist_v = [], []
    sm, sv = 1.0, 1.0
    for t in range(1, 12):
        g = _grad(n, 300 + t, -6 + (t % 5), -1 + (t % 5))  # amax jumps around
        _step(st, g, t, ex=True, margin_m=1, margin_v=2, hist_len=H)
        if t == 1:
            src_m, src_v = float(st.amax_m[0]), float(st.amax_v[0])
        else:
            src_m, src_v = max(hist_m[-H:]), max(hist_v[-H:])
        sm = pins.pow2scale_bruteforce(E4M3, src_m, sm) / 2 if src_m > 0 else sm
        sv = pins.pow2scale_bruteforce(E5M2, src_v, sv) / 4 if src_v > 0 else sv
        assert float(st.scale_m[0]) == sm and float(st.scale_v[0]) == sv, t
        hist_m.append(float(st.amax_m[0]))
        hist_v.append(float(st.amax_v[0]))
        assert st.hist_m[(t - 1) % H] == np.float32(hist_m[-1])
    # the ring holds the last H amax values
    assert sorted(st.hist_m.tolist()) == sorted(np.float32(hist_m[-H:]).tolist())


def test_update_from_stored_moments_closed_form(orc):
    """The update reads dec(code)/scale: p' = p*decay - step_size *
    m_q / (sqrt(v_q)*isbc2 + eps), with m_q, v_q the stored moments."""
    n = 4000
    rng = np.random.default_rng(12)
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    for fmts in ((E4M3, E5M2), (E4M3, E4M3)):
        st = orc.TensorState(p0, *fmts)
        for t in range(1, 5):
            g = _grad(n, 400 + t)
            p_before = st.p.astype(np.float64)
            _step(st, g, t, ex=True, flags=orc.FLAG_UPDATE_FROM_STORED)
            mq = orc.decode(fmts[0], st.m).astype(np.float64) / float(st.scale_m[0])
            vq = orc.decode(fmts[1], st.v).astype(np.float64) / float(st.scale_v[0])
            c = orc.step_constants(HP["lr"], HP["beta1"], HP["beta2"], HP["eps"], HP["wd"], t).astype(np.float64)
            exp = p_before * c[7] - c[4] * mq / (np.sqrt(vq) * c[5] + c[6])
            assert pins.params_close(st.p, exp, HP["lr"], 1, p_before=p_before)
        if fmts[1] == E4M3:
            # v flushed to 0 while m is not: the update is m/eps, far above lr
            # (the explainer's "1/(0+eps)" case)
            blown = (st.v & 0x7F == 0) & (st.m & 0x7F != 0)
            assert blown.any()
            dp = np.abs(st.p - p_before * c[7])
            assert np.allclose(dp[blown], c[4] * np.abs(mq[blown]) / c[6], rtol=1e-5)
            assert np.median(dp[blown]) > 100 * HP["lr"]


def test_grad_multiplier_power_of_two_equals_scaled_gradients(orc):
    n = 3000
    rng = np.random.default_rng(13)
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    a, b = orc.TensorState(p0, E4M3, E5M2), orc.TensorState(p0, E4M3, E5M2)
    for t in range(1, 5):
        g = _grad(n, 500 + t)
        g4 = _bf16_bits(pins.bf16_bits_to_f32(g) * 0.25)  # exact in bf16
        _step(a, g, t, ex=True, grad_mult=0.25)
        _step(b, g4, t)
        for x in ("p", "m", "v", "scale_m", "amax_v"):
            assert (getattr(a, x).view(np.uint8) == getattr(b, x).view(np.uint8)).all(), x


def test_grad_multiplier_matches_torch_adamw(orc):
    """Any multiplier c: torch.optim.AdamW on fp32 grads g*c, fp32 moments."""
    n = 3000
    rng = np.random.default_rng(14)
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    c = f32(0.3)
    st = orc.TensorState(p0, FP32, FP32)
    param = torch.nn.Parameter(torch.from_numpy(p0.copy()))
    opt = torch.optim.AdamW([param], lr=f32(HP["lr"]), betas=(f32(0.9), f32(0.95)), eps=f32(1e-8),
                            weight_decay=f32(0.1), foreach=False)
    for t in range(1, 6):
        g = _grad(n, 600 + t)
        _step(st, g, t, ex=True, grad_mult=c)
        param.grad = torch.from_numpy(pins.bf16_bits_to_f32(g) * np.float32(c))
        opt.step()
        assert pins.params_close(st.p, param.detach().numpy(), HP["lr"], t)


def test_skip_leaves_state_untouched_and_bf16_copy(orc):
    n = 1000
    rng = np.random.default_rng(15)
    st = orc.TensorState((rng.standard_normal(n) * 0.02).astype(np.float32), E4M3, E5M2)
    _step(st, _grad(n, 700), 1, ex=True, want_bf16=True)
    lib = torch.from_numpy(st.p.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert (st.p_bf16 == lib).all()
    snap = [x.copy() for x in (st.p, st.m, st.v, st.scale_m, st.amax_v)]
    _step(st, _grad(n, 701), 2, ex=True, skip=True)
    for a, b in zip(snap, (st.p, st.m, st.v, st.scale_m, st.amax_v)):
        assert (a.view(np.uint8) == b.view(np.uint8)).all()


def test_stochastic_rounding_step_codes(orc):
    """With stochastic rounding every code is one of the two grid neighbours
    of the value the deterministic step would round, drawn with the
    element's own Philox bits (recomputed here per element)."""
    n = 2000
    rng = np.random.default_rng(16)
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    sr = orc.TensorState(p0, E4M3, E5M2)
    fp = orc.TensorState(p0, FP32, FP32)
    seed, ti = 0x1234_5678_9ABC, 3
    g = _grad(n, 800)
    _step(sr, g, 1, ex=True, flags=orc.FLAG_STOCHASTIC, seed=seed, tensor_index=ti)
    _step(fp, g, 1)
    # step 1 from zero state: the unquantised moments equal the fp32 run's
    for fmt, q, x, s, which in ((E4M3, sr.m, fp.m, sr.scale_m, 0), (E5M2, sr.v, fp.v, sr.scale_v, 1)):
        xs = (x * s[0]).astype(np.float32)
        for j in range(n):
            r = orc.sr_bits(seed, ti, 1, j, which)
            assert q[j] == orc.encode_sr(fmt, float(xs[j]), r)
    # the update itself does not depend on the rounding mode (R2)
    assert (sr.p.view(np.uint32) == fp.p.view(np.uint32)).all()


@pytest.mark.parametrize("fmt", [E4M3, E5M2], ids=["e4m3", "e5m2"])
def test_sr_threshold_is_exact(orc, fmt):
    """At the draw r = T - 1 the oracle rounds up to hi, at r = T down to lo,
    T = ceil((|x|-lo)/(hi-lo) * 2^32) computed in float64 from the torch
    float8 grid; out of range and non-finite inputs saturate or give NaN."""
    x, r, want_up = pins.sr_cases(fmt, 17)
    got = orc.encode_sr_array(fmt, x, r)
    decided = want_up >= 0
    lo, hi, _ = pins.sr_threshold(fmt, x[decided])
    val = np.abs(orc.decode(fmt, got[decided] & 0x7F).astype(np.float64))
    assert (val == np.where(want_up[decided] == 1, hi, lo)).all()
    assert ((got[decided] >> 7) == np.signbit(x[decided])).all()
    # every code is one of the two neighbours (or the saturated / NaN code)
    fin = np.isfinite(x) & (np.abs(x) < pins.FMAX[fmt])
    lo, hi, _ = pins.sr_threshold(fmt, np.where(fin, x, 0.0))
    v = np.abs(orc.decode(fmt, got & 0x7F).astype(np.float64))
    assert ((v == lo) | (v == hi))[fin].all()
    big = ~np.isnan(x) & (np.abs(x) >= pins.FMAX[fmt])
    assert (v[big] == pins.FMAX[fmt]).all()
    assert ((got[np.isnan(x)] & 0x7F) == 0x7F).all()
    # the array form is the scalar encoder element by element
    for j in range(0, x.size, 97):
        assert got[j] == orc.encode_sr(fmt, float(x[j]), int(r[j]))
