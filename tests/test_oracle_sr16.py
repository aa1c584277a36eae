"""Pins of the oracle's stochastic rounding with 16-bit draws (CPU).

The rule (a reading of "随机舍入" in the strategy list of "FP8训练的稳定性挑战…",
which fixes neither generator nor resolution): code k of four takes a 16-bit
draw r from a 32-bit word (low half, low half bit-reversed, high half, high
half bit-reversed) and rounds up iff floor((|x|-lo)/(hi-lo) * 2^16) + r >= 2^16.

The encoder is checked against float64 thresholds on the torch float8 grid,
against the closed-form count of rounding-up draws over all 2^16 draws, and
against the 32-bit stochastic-rounding encoder, which it reproduces exactly
wherever (|x|-lo)/(hi-lo) has at most 32 fractional bits.  The draw counter
is checked against the Philox4x32-10 known-answer-pinned generator.  The lane
order is the device conversion's; the GPU codec tests check it against that
instruction on every fp32 input.
"""
import numpy as np
import pytest

import pins
from pins import E4M3, E5M2, FP32, FMAX

HP = dict(lr=3e-4, beta1=0.9, beta2=0.95, eps=1e-8, wd=0.1)


def test_rev16_reverses_the_bit_order(orc):
    for x in range(0, 1 << 16, 7):
        want = int(format(x, "016b")[::-1], 2)
        assert orc.rev16(x) == want
    assert orc.rev16(0x0001) == 0x8000 and orc.rev16(0x00FF) == 0xFF00 and orc.rev16(0xFFFF) == 0xFFFF


def test_sr16_draw_lanes(orc):
    """Codes 0 and 2 take the low and high halves of the word, codes 1 and 3
    the same halves with their bits in reverse order."""
    rng = np.random.default_rng(3)
    for w in [0, 0xFFFFFFFF, 0x00010000, 0x00000001, 0x80000000] + [int(v) for v in rng.integers(0, 1 << 32, 200)]:
        lo, hi = w & 0xFFFF, w >> 16
        assert orc.sr16_draw(w, 0) == lo
        assert orc.sr16_draw(w, 2) == hi
        assert orc.sr16_draw(w, 1) == int(format(lo, "016b")[::-1], 2)
        assert orc.sr16_draw(w, 3) == int(format(hi, "016b")[::-1], 2)


def _cases(fmt, seed):
    """Adversarial inputs (the 32-bit encoder's cases) with 16-bit draws at the
    threshold: r = 2^16 - F rounds up, r = 2^16 - F - 1 down; plus random
    draws.  Returns (x, r16, want_up) with -1 where the draw is random."""
    x, _, _ = pins.sr_cases(fmt, seed)
    rng = np.random.default_rng(seed + 1)
    live = np.isfinite(x) & (np.abs(x) < FMAX[fmt])
    _, _, F = pins.sr16_threshold(fmt, np.where(live, x, 0.0))
    T = 65536.0 - F
    xs, rs, up = [], [], []
    for sel, u in ((T, 1), (T - 1, 0)):
        ok = live & (sel >= 0) & (sel <= 65535)
        xs.append(x[ok])
        rs.append(sel[ok].astype(np.uint32))
        up.append(np.full(int(ok.sum()), u, np.int8))
    xs.append(x)
    rs.append(rng.integers(0, 1 << 16, x.size).astype(np.uint32))
    up.append(np.full(x.size, -1, np.int8))
    return np.concatenate(xs).astype(np.float32), np.concatenate(rs), np.concatenate(up)


@pytest.mark.parametrize("fmt", [E4M3, E5M2], ids=["e4m3", "e5m2"])
def test_sr16_threshold_is_exact(orc, fmt):
    """At r = 2^16 - F the oracle rounds up to hi, one below it down to lo
    (F from float64 on the torch float8 grid); every code is one of the two
    neighbours, the sign is kept, |x| >= max saturates, NaN gives 0x7F."""
    x, r, want_up = _cases(fmt, 29)
    got = orc.encode_sr16_array(fmt, x, r)
    dec = want_up >= 0
    lo, hi, _ = pins.sr16_threshold(fmt, x[dec])
    val = np.abs(orc.decode(fmt, got[dec] & 0x7F).astype(np.float64))
    assert (val == np.where(want_up[dec] == 1, hi, lo)).all()
    assert ((got[dec] >> 7) == np.signbit(x[dec])).all()
    fin = np.isfinite(x) & (np.abs(x) < FMAX[fmt])
    lo, hi, _ = pins.sr16_threshold(fmt, np.where(fin, x, 0.0))
    v = np.abs(orc.decode(fmt, got & 0x7F).astype(np.float64))
    assert ((v == lo) | (v == hi))[fin].all()
    big = ~np.isnan(x) & (np.abs(x) >= FMAX[fmt])
    assert (v[big] == FMAX[fmt]).all()
    assert ((got[big] >> 7) == np.signbit(x[big])).all()
    assert (got[np.isnan(x)] == 0x7F).all()
    for j in range(0, x.size, 101):
        assert got[j] == orc.encode_sr16(fmt, float(x[j]), int(r[j]))


@pytest.mark.parametrize("fmt", [E4M3, E5M2], ids=["e4m3", "e5m2"])
def test_sr16_counts_of_rounding_up_over_all_draws(orc, fmt):
    """Over all 2^16 draws exactly F = floor((|x|-lo)/(hi-lo) * 2^16) round up
    (closed form), so the mean code value is lo + (hi-lo) * F / 2^16: biased
    toward zero by less than (hi-lo) * 2^-16."""
    rng = np.random.default_rng(31)
    grid = pins.finite_grid(fmt)
    xs = np.concatenate([
        (rng.standard_normal(150) * 10.0 ** rng.uniform(-7, 2.5, 150)),
        (grid[1:-1] + grid[:-2]) / 2,                         # midpoints
        grid[1:-1][::9] + np.diff(grid)[1:][::9] * 2.0 ** -17,  # just above grid values
        grid[1:-1][::9],                                         # grid values
    ]).astype(np.float32)
    xs = xs[np.isfinite(xs) & (np.abs(xs) < FMAX[fmt])]
    r = np.arange(1 << 16, dtype=np.uint32)
    for x in xs:
        codes = orc.encode_sr16_array(fmt, np.full(r.size, x, np.float32), r)
        lo, hi, F = pins.sr16_threshold(fmt, np.array([x]))
        v = np.abs(orc.decode(fmt, codes & 0x7F).astype(np.float64))
        n_up = int((v == hi[0]).sum())
        assert n_up == int(F[0]), (x, n_up, F[0])
        assert int((v == lo[0]).sum()) == r.size - n_up
        # the draws that round up are the top F ones
        assert n_up == 0 or (v[r >= (1 << 16) - n_up] == hi[0]).all()
        mean = lo[0] + (hi[0] - lo[0]) * n_up / 65536.0  # exact in float64
        assert 0.0 <= abs(float(x)) - mean < (hi[0] - lo[0]) * 2.0 ** -16


@pytest.mark.parametrize("fmt", [E4M3, E5M2], ids=["e4m3", "e5m2"])
def test_sr16_is_the_32_bit_encoder_at_expanded_draws(orc, fmt):
    """The 32-bit encoder rounds up iff r32 < (|x|-lo)/(hi-lo) * 2^32.  With
    r32 = (2^16 - r16) * 2^16 - 1 that is the 16-bit rule whenever
    (|x|-lo)/(hi-lo) * 2^32 is an integer: |x| >= 2^-18 (E4M3) or 2^-25 (E5M2),
    every normal and subnormal grid interval included."""
    rng = np.random.default_rng(37)
    low_e = -18 if fmt == E4M3 else -25
    e = rng.integers(low_e, 17, 20000)
    mant = rng.integers(0, 1 << 23, 20000)
    bits = (((127 + e).astype(np.uint64) << 23) | mant.astype(np.uint64)).astype(np.uint32)
    x = bits.view(np.float32)
    x = np.where(rng.integers(0, 2, x.size) == 1, -x, x).astype(np.float32)
    r16 = rng.integers(0, 1 << 16, x.size).astype(np.uint32)
    # threshold draws too
    live = np.abs(x) < FMAX[fmt]
    _, _, F = pins.sr16_threshold(fmt, np.where(live, x, 0.0))
    r16 = np.where(rng.integers(0, 2, x.size) == 1, np.clip(65536 - F, 0, 65535), r16).astype(np.uint32)
    r32 = ((65535 - r16.astype(np.uint64)) << 16 | 0xFFFF).astype(np.uint32)
    assert (orc.encode_sr16_array(fmt, x, r16) == orc.encode_sr_array(fmt, x, r32)).all()


def test_sr16_words_form(orc):
    """encode_sr16_words takes code j's draw from lane j % 4 of word j // 4."""
    rng = np.random.default_rng(41)
    x = (rng.standard_normal(4000) * 10.0 ** rng.uniform(-6, 2, 4000)).astype(np.float32)
    w = rng.integers(0, 1 << 32, 1000, dtype=np.uint64).astype(np.uint32)
    for fmt in (E4M3, E5M2):
        got = orc.encode_sr16_words(fmt, x, w)
        r16 = np.array([orc.sr16_draw(int(w[j // 4]), j % 4) for j in range(x.size)], np.uint32)
        assert (got == orc.encode_sr16_array(fmt, x, r16)).all()


def test_sr16_bits_counter(orc):
    """One Philox4x32-10 call (known-answer pinned) per eight elements: counter
    (j/8, tensor, step), key = seed; outputs 0/1 serve m/v of elements
    8q..8q+3, outputs 2/3 those of 8q+4..8q+7, code j % 4 of the word."""
    seed, ti, t = 0x0123_4567_89AB_CDEF, 5, 9
    for j in list(range(0, 64)) + [8 * 12345 + k for k in range(8)] + [(1 << 33) + 8 + k for k in range(8)]:
        q = j >> 3
        out = orc.philox4x32_10([q & 0xFFFFFFFF, q >> 32, ti, t], [seed & 0xFFFFFFFF, seed >> 32])
        for which in (0, 1):
            w = out[2 * ((j >> 2) & 1) + which]
            assert orc.sr16_bits(seed, ti, t, j, which) == orc.sr16_draw(w, j & 3)


def test_sr16_draws_are_uniform_and_vary(orc):
    vals = np.array([orc.sr16_bits(7, 3, 5, j, w) for j in range(8192) for w in (0, 1)], np.int64)
    assert vals.min() >= 0 and vals.max() < 1 << 16
    hist = np.bincount(vals >> 8, minlength=256)
    exp = vals.size / 256
    assert ((hist - exp) ** 2 / exp).sum() < 400  # chi-square, 255 dof
    same = sum(orc.sr16_bits(7, 3, 5, j, 0) == orc.sr16_bits(7, 3, 6, j, 0) for j in range(256))
    assert same < 8  # a new draw each step
    same = sum(orc.sr16_bits(7, 3, 5, j, 0) == orc.sr16_bits(8, 3, 5, j, 0) for j in range(256))
    assert same < 8  # and per seed


def test_sr16_step_codes(orc):
    """With 16-bit-draw stochastic rounding every code equals the encoder's at
    the element's own draw (recomputed here per element); the update itself
    does not depend on the rounding (the update reads the unquantised
    moments)."""
    n = 2003
    rng = np.random.default_rng(43)
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    sr = orc.TensorState(p0, E4M3, E5M2)
    fp = orc.TensorState(p0, FP32, FP32)
    seed, ti = 0x1234_5678_9ABC, 3
    g = (rng.standard_normal(n) * 10.0 ** rng.uniform(-6, -1, n)).astype(np.float32)
    import torch
    gb = torch.from_numpy(g).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    sr.step_ex(gb, HP["lr"], HP["beta1"], HP["beta2"], HP["eps"], HP["wd"], 1,
               orc.FLAG_STOCHASTIC | orc.FLAG_SR_DRAW16, seed=seed, tensor_index=ti)
    fp.step(gb, HP["lr"], HP["beta1"], HP["beta2"], HP["eps"], HP["wd"], 1, 0)
    for fmt, q, x, s, which in ((E4M3, sr.m, fp.m, sr.scale_m, 0), (E5M2, sr.v, fp.v, sr.scale_v, 1)):
        xs = (x * s[0]).astype(np.float32)
        for j in range(n):
            assert q[j] == orc.encode_sr16(fmt, float(xs[j]), orc.sr16_bits(seed, ti, 1, j, which))
    assert (sr.p.view(np.uint32) == fp.p.view(np.uint32)).all()
    # the 32-bit rule gives other codes from the same seed
    sr32 = orc.TensorState(p0, E4M3, E5M2)
    sr32.step_ex(gb, HP["lr"], HP["beta1"], HP["beta2"], HP["eps"], HP["wd"], 1, orc.FLAG_STOCHASTIC,
                 seed=seed, tensor_index=ti)
    assert (sr32.m != sr.m).any()
