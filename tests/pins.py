"""Independent references the oracle is pinned to (test code only).

* ``torch_encode``: PyTorch's own float8 casts (a library routine), valid for
  |x| <= max of the format (torch does not saturate the way satfinite does).
* ``rint_encode``: a second round-to-nearest-even encoder written from the
  format definition in float64 numpy (frexp/ldexp/rint); it shares no code
  with the oracle, which searches a table of decoded values.
* ``pow2scale_bruteforce``: the largest 2^k (|k| <= 126) with amax*2^k <= max,
  found by trying every k.
* ``TorchFakeQuantAdamW``: ``torch.optim.AdamW`` (a library routine) whose
  moments are stored between steps as power-of-two-scaled float8 via the
  torch casts above.
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch

E4M3, E5M2, FP32 = 0, 1, 2
FMAX = {E4M3: 448.0, E5M2: 57344.0}
TORCH_DT = {E4M3: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}
GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def f32(x) -> float:
    """Round a Python float to the nearest fp32 value."""
    return float(np.float32(x))


def params_close(p, p_ref, lr: float, steps: int, rtol: float = 1e-6, p_before=None) -> bool:
    """|p - p_ref| <= rtol * (|p_ref| + U), U the size of the update(s).

    Params that pass near zero make p*decay - step_size*u cancel, and a large
    m/sqrt(v) makes the update itself large: either way the rounding error is
    relative to the update, not to p.  U = |p_ref - p_before| when the params
    before the step are given, plus lr*steps (the typical update scale)."""
    p = np.asarray(p, np.float64)
    p_ref = np.asarray(p_ref, np.float64)
    u = lr * steps
    if p_before is not None:
        u = u + np.abs(p_ref - np.asarray(p_before, np.float64))
    return bool((np.abs(p - p_ref) <= rtol * (np.abs(p_ref) + u)).all())


# ------------------------------------------------------------------ codec
def torch_encode(fmt: int, x: torch.Tensor) -> torch.Tensor:
    return x.to(TORCH_DT[fmt]).view(torch.uint8)


def torch_decode(fmt: int, codes: torch.Tensor) -> torch.Tensor:
    return codes.view(TORCH_DT[fmt]).to(torch.float32)


def rint_encode(fmt: int, x: np.ndarray) -> np.ndarray:
    """RNE + satfinite encode written from the format definition with float64
    arithmetic: split |x| = m * 2^e (frexp), take the quantum of its binade
    (2^(max(e-1, emin) - M)), count quanta with np.rint (round half to even)
    and assemble exponent and mantissa fields.  NaN -> 0x7F."""
    M = 3 if fmt == E4M3 else 2
    bias = 7 if fmt == E4M3 else 15
    emin = 1 - bias
    maxcode = 0x7E if fmt == E4M3 else 0x7B
    x = np.asarray(x, np.float32)
    a = np.abs(x).astype(np.float64)
    with np.errstate(invalid="ignore", over="ignore"):
        _, e = np.frexp(a)                             # frexp(0) gives e = 0
        eb = np.maximum(np.where(a > 0, e - 1, emin), emin)  # binade exponent (>= emin)
        n = np.rint(np.ldexp(a, M - eb))               # quanta of 2^(eb-M), exact scaling
        n = np.where(np.isfinite(n), n, 0.0)
        code = ((eb - emin).astype(np.int64) << M) + n.astype(np.int64)
    code = np.minimum(code, maxcode)
    code = np.where(np.isinf(a), maxcode, code)
    code = code | np.where(np.signbit(x), 0x80, 0)
    code = np.where(np.isnan(x), 0x7F, code)
    return code.astype(np.uint8)


def load_runs(fmt: int):
    name = "e4m3" if fmt == E4M3 else "e5m2"
    starts, codes = [], []
    with open(os.path.join(GOLDEN, "codec_runs_%s.txt" % name)) as f:
        for line in f:
            if line.startswith("#"):
                continue
            a, b = line.split()
            starts.append(int(a, 16))
            codes.append(int(b, 16))
    return np.array(starts, np.int64), np.array(codes, np.uint8)


def expand_runs(starts: np.ndarray, codes: np.ndarray, first: int, n: int) -> np.ndarray:
    """Codes of bit patterns first .. first+n-1 from a run table."""
    ends = np.append(starts[1:], 1 << 32)
    lo, hi = first, first + n
    i0 = np.searchsorted(starts, lo, side="right") - 1
    i1 = np.searchsorted(starts, hi, side="left")
    s = np.clip(starts[i0:i1], lo, hi)
    e = np.clip(ends[i0:i1], lo, hi)
    return np.repeat(codes[i0:i1], (e - s).astype(np.int64))


# ------------------------------------------------------------------ scale
def pow2scale_bruteforce(fmt: int, amax: float, s_prev: float) -> float:
    if not math.isfinite(amax) or not amax > 0:
        return s_prev
    best = None
    for k in range(-126, 127):
        if amax * 2.0 ** k <= FMAX[fmt]:
            best = k
    if best is None:
        best = -126
    return 2.0 ** best


# ------------------------------------------------------------------ step
def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


class TorchFakeQuantAdamW:
    """One-tensor AdamW via torch.optim.AdamW, moments held between steps as
    float8 codes with power-of-two per-tensor scales (delayed scaling with the
    previous step's amax; step 1 uses its own amax)."""

    def __init__(self, p: np.ndarray, m_fmt: int, v_fmt: int, lr, beta1, beta2, eps, wd):
        self.param = torch.nn.Parameter(torch.from_numpy(p.astype(np.float32).copy()))
        self.m_fmt, self.v_fmt = m_fmt, v_fmt
        self.hp = dict(lr=f32(lr), betas=(f32(beta1), f32(beta2)), eps=f32(eps),
                       weight_decay=f32(wd))
        n = p.size
        self.mq = torch.zeros(n, dtype=torch.uint8) if m_fmt != FP32 else torch.zeros(n)
        self.vq = torch.zeros(n, dtype=torch.uint8) if v_fmt != FP32 else torch.zeros(n)
        self.scale_m = 1.0
        self.scale_v = 1.0
        self.amax_m = 0.0
        self.amax_v = 0.0
        self.t = 0

    def _deq(self, fmt, q, s):
        if fmt == FP32:
            return q.clone()
        return torch_decode(fmt, q) * (1.0 / s)

    def step(self, g_bits: np.ndarray, jit_every_step: bool = False):
        self.t += 1
        opt = torch.optim.AdamW([self.param], foreach=False, fused=False, **self.hp)
        st = opt.state[self.param]
        st["step"] = torch.tensor(float(self.t - 1))
        st["exp_avg"] = self._deq(self.m_fmt, self.mq, self.scale_m)
        st["exp_avg_sq"] = self._deq(self.v_fmt, self.vq, self.scale_v)
        self.param.grad = torch.from_numpy(bf16_bits_to_f32(g_bits))
        opt.step()
        m_new, v_new = st["exp_avg"], st["exp_avg_sq"]
        am = float(m_new.abs().max()) if m_new.numel() else 0.0
        av = float(v_new.abs().max()) if v_new.numel() else 0.0
        if self.t == 1 or jit_every_step:
            prev_m, prev_v = am, av
        else:
            prev_m, prev_v = self.amax_m, self.amax_v
        if self.m_fmt != FP32:
            self.scale_m = pow2scale_bruteforce(self.m_fmt, prev_m, self.scale_m)
            self.mq = torch_encode(self.m_fmt, (m_new * self.scale_m).clamp(-FMAX[self.m_fmt], FMAX[self.m_fmt]))
        else:
            self.mq = m_new.clone()
        if self.v_fmt != FP32:
            self.scale_v = pow2scale_bruteforce(self.v_fmt, prev_v, self.scale_v)
            self.vq = torch_encode(self.v_fmt, (v_new * self.scale_v).clamp(-FMAX[self.v_fmt], FMAX[self.v_fmt]))
        else:
            self.vq = v_new.clone()
        self.amax_m, self.amax_v = am, av
        self.m_unq, self.v_unq = m_new.clone(), v_new.clone()
        return self

    @property
    def p(self) -> np.ndarray:
        return self.param.detach().numpy()


# ------------------------------------------------------------------ stochastic rounding
def finite_grid(fmt: int) -> np.ndarray:
    """The format's non-negative finite values in increasing order, from the
    torch float8 casts (codes 0x00..0x7F, NaN and inf dropped)."""
    vals = torch_decode(fmt, torch.arange(128, dtype=torch.int32).to(torch.uint8)).numpy().astype(np.float64)
    return np.unique(vals[np.isfinite(vals)])


def sr_threshold(fmt: int, x: np.ndarray):
    """For finite |x| below the format's max: (lo, hi, T) with lo <= |x| < hi
    neighbours on the grid and T = ceil((|x| - lo) / (hi - lo) * 2^32), the
    number of random words r that round |x| up (r < T).  float64 is exact
    here: |x| - lo has at most 24 significant bits and hi - lo is a power of
    two."""
    grid = finite_grid(fmt)
    a = np.abs(np.asarray(x, np.float64))
    k = np.searchsorted(grid, a, side="right") - 1
    lo, hi = grid[k], grid[k + 1]
    t = np.ceil((a - lo) / (hi - lo) * 4294967296.0)
    return lo, hi, t


def sr_cases(fmt: int, seed: int):
    """Adversarial inputs for a stochastic-rounding encoder: every fp32
    binade from the subnormals to beyond the format's max (edge and random
    mantissas, both signs), the grid values and their midpoints, and the
    specials; each finite in-range input with the draws r = T-1 (rounds up),
    r = T (rounds down) and a random r.  Returns (x, r, want_up) with want_up
    1/0 where the draw decides it and -1 elsewhere."""
    rng = np.random.default_rng(seed)
    bits = []
    for e in range(0, 146):
        mant = np.concatenate([[0, 1, 2, 0x3FFFFF, 0x400000, 0x400001, 0x7FFFFE, 0x7FFFFF],
                               rng.integers(0, 1 << 23, 24)])
        bits.append((e << 23) | mant)
    bits = np.concatenate(bits).astype(np.uint32)
    grid = finite_grid(fmt)
    extra = np.concatenate([grid, (grid[1:] + grid[:-1]) / 2, [FMAX[fmt], np.nextafter(np.float32(FMAX[fmt]), 0)]])
    x = np.concatenate([bits.view(np.float32), extra.astype(np.float32)])
    x = np.concatenate([x, -x])
    fmax = FMAX[fmt]
    live = np.isfinite(x) & (np.abs(x) < fmax)
    xs, rs, up = [], [], []
    _, _, t = sr_threshold(fmt, np.where(live, x, 0.0))
    for sel_r, u in ((t - 1, 1), (t, 0)):
        ok = live & (sel_r >= 0) & (sel_r <= 0xFFFFFFFF)
        xs.append(x[ok])
        rs.append(sel_r[ok].astype(np.uint64).astype(np.uint32))
        up.append(np.full(int(ok.sum()), u, np.int8))
    xs.append(x)
    rs.append(rng.integers(0, 1 << 32, x.size, dtype=np.uint64).astype(np.uint32))
    up.append(np.full(x.size, -1, np.int8))
    spec = np.array([np.nan, -np.nan, np.inf, -np.inf, 0.0, -0.0, 1e30, -1e30], np.float32)
    xs.append(spec)
    rs.append(rng.integers(0, 1 << 32, spec.size, dtype=np.uint64).astype(np.uint32))
    up.append(np.full(spec.size, -1, np.int8))
    return np.concatenate(xs).astype(np.float32), np.concatenate(rs), np.concatenate(up)


def sr16_threshold(fmt: int, x: np.ndarray):
    """For finite |x| below the format's max: (lo, hi, F) with lo <= |x| < hi
    neighbours on the torch float8 grid and F = floor((|x| - lo) / (hi - lo) *
    2^16); a 16-bit draw r rounds up iff F + r >= 2^16.  float64 is exact as
    in sr_threshold."""
    grid = finite_grid(fmt)
    a = np.abs(np.asarray(x, np.float64))
    k = np.searchsorted(grid, a, side="right") - 1
    lo, hi = grid[k], grid[k + 1]
    return lo, hi, np.floor((a - lo) / (hi - lo) * 65536.0)
