"""Pins of the oracle's FP8 codec (CPU).

The oracle's encode/decode are checked against things other than itself:
PyTorch's float8 casts (a library routine), a second encoder written from
the format definition, the values the pages print (format table, E4M3 smallest normal
~2^-6 ~ 0.0156, maxima), the closed form, and exhaustive agreement on all 2^32
fp32 inputs.  The run-length fixture written by
``tests/golden/make_codec_runs.py`` (oracle only) is checked here too.
"""
import json
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import pins


def test_all_codes_decode_like_torch(orc):
    """All 256 codes of each format: oracle decode == torch float8 -> fp32."""
    codes = np.arange(256, dtype=np.uint8)
    for fmt in (orc.E4M3, orc.E5M2):
        ours = orc.decode(fmt, codes)
        lib = pins.torch_decode(fmt, torch.from_numpy(codes)).numpy()
        nan_o, nan_l = np.isnan(ours), np.isnan(lib)
        assert (nan_o == nan_l).all()
        assert (ours[~nan_o].view(np.uint32) == lib[~nan_l].view(np.uint32)).all()


def test_format_layout_and_special_codes(orc):
    """Bit layouts of the format tables (E4M3: 4 exponent, 3 mantissa bits;
    E5M2: 5, 2), special codes and extreme values."""
    d4 = lambda c: float(orc.lib().ref_decode(orc.E4M3, c))
    d5 = lambda c: float(orc.lib().ref_decode(orc.E5M2, c))
    # E4M3: bias 7, no infinity, S.1111.111 NaN, max 0x7E = 448
    assert d4(0x38) == 1.0 and d4(0x40) == 2.0 and d4(0x39) == 1.125
    assert d4(0x7E) == 448.0 and math.isnan(d4(0x7F)) and math.isnan(d4(0xFF))
    assert d4(0x01) == 2.0 ** -9 and d4(0x08) == 2.0 ** -6
    assert d4(0x80) == 0.0 and math.copysign(1.0, d4(0x80)) == -1.0
    # E5M2: bias 15, 0x7C infinity, 0x7D..0x7F NaN, max 0x7B = 57344
    assert d5(0x3C) == 1.0 and d5(0x3D) == 1.25
    assert d5(0x7B) == 57344.0 and d5(0x7C) == math.inf and d5(0xFC) == -math.inf
    assert all(math.isnan(d5(c)) for c in (0x7D, 0x7E, 0x7F, 0xFD, 0xFE, 0xFF))
    assert d5(0x01) == 2.0 ** -16 and d5(0x04) == 2.0 ** -14
    assert orc.fmax(orc.E4M3) == 448.0 and orc.fmax(orc.E5M2) == 57344.0


def test_finite_codes_round_trip(orc):
    codes = np.arange(256, dtype=np.uint8)
    for fmt, nfinite in ((orc.E4M3, 254), (orc.E5M2, 248)):
        vals = orc.decode(fmt, codes)
        fin = np.isfinite(vals)
        assert fin.sum() == nfinite
        back = orc.encode(fmt, vals[fin])
        assert (back == codes[fin]).all()
    # infinities saturate to the largest finite code of the same sign
    assert orc.encode(orc.E5M2, np.array([np.inf, -np.inf], np.float32)).tolist() == [0x7B, 0xFB]
    assert orc.encode(orc.E4M3, np.array([np.inf, -np.inf], np.float32)).tolist() == [0x7E, 0xFE]


def test_ties_and_saturation(orc):
    E4, E5 = orc.E4M3, orc.E5M2
    x = np.array([2.0 ** -10, -(2.0 ** -10), 1.5 * 2.0 ** -9, 1.0625, 1.1875, 449.0, 463.9, 464.0,
                  1e30, -1e30, 0.0, -0.0], np.float32)
    got = orc.encode(E4, x).tolist()
    # 2^-10 is half the smallest subnormal: tie -> even code 0 (sign kept);
    # 1.0625 = midpoint of 1 (0x38) and 1.125 (0x39) -> 0x38; 1.1875 -> 0x3A
    assert got == [0x00, 0x80, 0x02, 0x38, 0x3A, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x00, 0x80]
    y = np.array([57344.0, 61440.0, 1e9, 2.0 ** -17, 3 * 2.0 ** -17, 1.125, 1.375], np.float32)
    # 2^-17 = half of 2^-16 -> 0; 3*2^-17 -> tie between 1 and 2 -> 2;
    # 1.125 midpoint of 1.0 (0x3C) and 1.25 (0x3D) -> 0x3C; 1.375 -> 0x3E
    assert orc.encode(E5, y).tolist() == [0x7B, 0x7B, 0x7B, 0x00, 0x02, 0x3C, 0x3E]
    # NaN of either sign and any payload -> 0x7F in both formats.  The pages
    # are silent on the sign of a NaN code; this reading follows the B200's
    # cvt.rn.satfinite conversion, which the exhaustive device test checks on
    # every NaN input (torch's CPU cast would keep the sign: 0xFF for -NaN)
    nans = np.array([0x7FC00000, 0xFFC00000, 0x7F800001, 0xFF800001, 0x7FFFFFFF, 0xFFFFFFFF],
                    np.uint32).view(np.float32)
    assert (orc.encode(E4, nans) == 0x7F).all() and (orc.encode(E5, nans) == 0x7F).all()
    assert all(orc.encode_sr(f, float(x), r) == 0x7F for f in (E4, E5) for x in nans for r in (0, 2 ** 32 - 1))


def test_worked_example_from_the_pages(orc):
    """The pages' numeric example of why v is stored in E5M2."""
    with open(os.path.join(pins.GOLDEN, "worked_example.json")) as f:
        ex = json.load(f)
    v_a = ex["v_A"]
    # E5M2 keeps 1e-4: 1/sqrt(v) ~ 100
    q5 = orc.encode(orc.E5M2, np.array([v_a], np.float32))[0]
    r5 = 1.0 / math.sqrt(float(orc.decode(orc.E5M2, [q5])[0]))
    assert q5 == 0x07
    assert abs(r5 - ex["inv_sqrt_e5m2_approx"]) / ex["inv_sqrt_e5m2_approx"] < ex["rel_tol_approx"]
    # E4M3 flushes it to zero ...
    q4 = orc.encode(orc.E4M3, np.array([v_a], np.float32))[0]
    assert q4 == 0x00
    assert float(orc.decode(orc.E4M3, [q4])[0]) == 0.0
    # ... its smallest normal is ~2^-6 ~ 0.0156, and snapping there gives 8
    mn = float(orc.decode(orc.E4M3, [0x08])[0])
    assert mn == 2.0 ** ex["e4m3_min_normal_log2"]
    assert abs(mn - ex["e4m3_min_normal_approx"]) < 1e-4
    assert 1.0 / math.sqrt(mn) == ex["inv_sqrt_snapped"]
    assert round(ex["inv_sqrt_e5m2_approx"] / ex["inv_sqrt_snapped"]) == ex["error_factor"]
    # v_B = 1 is exact in both formats
    for fmt in (orc.E4M3, orc.E5M2):
        assert float(orc.decode(fmt, orc.encode(fmt, np.array([ex["v_B"]], np.float32)))[0]) == 1.0
    # E5M2 reaches both smaller and larger values than E4M3
    assert orc.decode(orc.E5M2, [1])[0] < orc.decode(orc.E4M3, [1])[0]
    assert orc.fmax(orc.E5M2) > orc.fmax(orc.E4M3)


def test_fixture_matches_oracle_on_boundaries_and_sample(orc):
    rng = np.random.default_rng(7)
    for fmt in (orc.E4M3, orc.E5M2):
        starts, codes = pins.load_runs(fmt)
        probe = np.unique(np.clip(np.concatenate([starts - 1, starts, starts + 1]), 0, (1 << 32) - 1))
        bits = np.concatenate([probe, rng.integers(0, 1 << 32, size=1 << 20, dtype=np.int64)])
        x = bits.astype(np.uint32).view(np.float32)
        exp = np.concatenate([pins.expand_runs(starts, codes, int(b), 1) for b in bits[:len(probe)]])
        got = orc.encode(fmt, x)
        assert (got[:len(probe)] == exp).all()
        idx = np.searchsorted(starts, bits[len(probe):], side="right") - 1
        assert (got[len(probe):] == codes[idx]).all()


def _exhaustive_chunk(orc, fmt, first, n):
    xn = np.arange(first, first + n, dtype=np.uint32).view(np.float32)
    x = torch.from_numpy(xn)
    ours = torch.from_numpy(orc.encode_bits_range(fmt, first, n))
    # (a) the independent float64/rint encoder, every input
    bw = torch.from_numpy(pins.rint_encode(fmt, xn))
    bad_bw = int((bw != ours).sum())
    # (b) torch's float8 cast where it is defined the same way (|x| <= max)
    inr = x.abs() <= pins.FMAX[fmt]
    lib = pins.torch_encode(fmt, torch.where(inr, x, torch.zeros_like(x)))
    bad_lib = int(((lib != ours) & inr).sum())
    # (c) the committed run-length fixture
    starts, codes = pins.load_runs(fmt)
    fx = torch.from_numpy(pins.expand_runs(starts, codes, first, n))
    bad_fx = int((fx != ours).sum())
    return bad_bw, bad_lib, bad_fx, int(inr.sum())


@pytest.mark.slow
@pytest.mark.parametrize("fmt", [0, 1], ids=["e4m3", "e5m2"])
def test_exhaustive_all_fp32_inputs(orc, fmt):
    """Every one of the 2^32 fp32 bit patterns: oracle == rint encoder
    == torch float8 cast (in range) == committed fixture."""
    chunk = 1 << 24
    threads = len(os.sched_getaffinity(0))
    torch.set_num_threads(1)
    try:
        with ThreadPoolExecutor(threads) as ex:
            res = list(ex.map(lambda f: _exhaustive_chunk(orc, fmt, f, chunk),
                              range(0, 1 << 32, chunk)))
    finally:
        torch.set_num_threads(threads)
    assert sum(r[0] for r in res) == 0
    assert sum(r[1] for r in res) == 0
    assert sum(r[2] for r in res) == 0
    assert sum(r[3] for r in res) > (1 << 30)  # the library pin covered >1/4 of all inputs
