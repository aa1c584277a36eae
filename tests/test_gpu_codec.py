"""Device FP8 codec against the oracle, through the C ABI.

Both device implementations (hardware cvt, integer path) must equal the
oracle on all 256 codes (decode) and, byte for byte, on all 2^32 fp32 inputs
(encode; the oracle's encoding of every input is the committed run-length
fixture written by tests/golden/make_codec_runs.py).  That includes the 2^24
NaN inputs of each format: the hardware conversion gives 0x7F for every NaN,
whatever its sign, and so do the oracle and the integer path.
"""
import numpy as np
import pytest
import torch

import oracle
import pins
from fp8_quantized_adam_b200 import capi

pytestmark = pytest.mark.gpu

IMPLS = [0, 1]
IMPL_IDS = ["hw", "sw"]


def _stream():
    return torch.cuda.current_stream().cuda_stream


@pytest.mark.parametrize("impl", IMPLS, ids=IMPL_IDS)
@pytest.mark.parametrize("fmt", [0, 1], ids=["e4m3", "e5m2"])
def test_decode_all_codes(fmt, impl):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8).cuda()
    out = torch.empty(256, dtype=torch.float32, device="cuda")
    capi.fp8adam_decode(fmt, codes.data_ptr(), out.data_ptr(), 256, impl, _stream())
    got = out.cpu().numpy()
    exp = oracle.decode(fmt, np.arange(256, dtype=np.uint8))
    nan = np.isnan(exp)
    assert (np.isnan(got) == nan).all()
    assert (got[~nan].view(np.uint32) == exp[~nan].view(np.uint32)).all()


@pytest.mark.slow
@pytest.mark.parametrize("impl", IMPLS, ids=IMPL_IDS)
@pytest.mark.parametrize("fmt", [0, 1], ids=["e4m3", "e5m2"])
def test_encode_all_fp32_inputs(fmt, impl):
    starts, codes = pins.load_runs(fmt)
    chunk = 1 << 28
    out = torch.empty(chunk, dtype=torch.uint8, device="cuda")
    bad = 0
    for first in range(0, 1 << 32, chunk):
        capi.fp8adam_encode_bits_range(fmt, first, chunk, out.data_ptr(), impl, _stream())
        got = out.cpu().numpy()
        exp = pins.expand_runs(starts, codes, first, chunk)
        bad += int((got != exp).sum())
    assert bad == 0


@pytest.mark.parametrize("impl", IMPLS, ids=IMPL_IDS)
@pytest.mark.parametrize("fmt", [0, 1], ids=["e4m3", "e5m2"])
def test_encode_array_ragged(fmt, impl):
    rng = np.random.default_rng(3)
    n = 100_003  # not a multiple of the 4 elements a thread takes
    x = (rng.standard_normal(n) * 10.0 ** rng.uniform(-12, 6, n)).astype(np.float32)
    x[:8] = [0.0, -0.0, np.inf, -np.inf, 448.0, 464.0, 57344.0, 61440.0]
    xd = torch.from_numpy(x).cuda()
    out = torch.empty(n, dtype=torch.uint8, device="cuda")
    capi.fp8adam_encode(fmt, xd.data_ptr(), out.data_ptr(), n, impl, _stream())
    assert (out.cpu().numpy() == oracle.encode(fmt, x)).all()


@pytest.mark.parametrize("fmt", [0, 1], ids=["e4m3", "e5m2"])
def test_stochastic_rounding_encoder(fmt):
    """The device SR encoder (the one the step uses with stochastic rounding)
    against the oracle on adversarial inputs: every fp32 binade, grid values
    and midpoints, specials, and for each in-range input the draws on both
    sides of its exact threshold."""
    x, r, _ = pins.sr_cases(fmt, 29)
    exp = oracle.encode_sr_array(fmt, x, r)
    dx = torch.from_numpy(x).cuda()
    dr = torch.from_numpy(r.view(np.int32)).cuda()
    out = torch.empty(x.size, dtype=torch.uint8, device="cuda")
    capi.fp8adam_encode_sr(fmt, dx.data_ptr(), dr.data_ptr(), out.data_ptr(), x.size, _stream())
    got = out.cpu().numpy()
    assert (got[np.isnan(x)] == 0x7F).all()  # NaN of either sign, as the hardware conversion
    d = np.flatnonzero(got != exp)
    assert d.size == 0, (x[d[:8]], r[d[:8]], got[d[:8]], exp[d[:8]])


def _sr16_words_for(r16: np.ndarray, lane: np.ndarray, rng) -> np.ndarray:
    """Words whose draw for code `lane` is r16 (the other half random)."""
    r = r16.astype(np.uint64)
    rev = np.zeros_like(r)
    for b in range(16):
        rev |= ((r >> np.uint64(b)) & np.uint64(1)) << np.uint64(15 - b)
    other = rng.integers(0, 1 << 16, r.size).astype(np.uint64)
    w = np.where(lane == 0, (other << 16) | r,
        np.where(lane == 1, (other << 16) | rev,
        np.where(lane == 2, (r << 16) | other, (rev << 16) | other)))
    return w.astype(np.uint32)


def _encode_sr16_device(fmt: int, x: np.ndarray, w: np.ndarray) -> np.ndarray:
    dx = torch.from_numpy(x).cuda()
    dw = torch.from_numpy(w.view(np.int32)).cuda()
    out = torch.full((x.size,), 0xAA, dtype=torch.uint8, device="cuda")
    capi.fp8adam_encode_sr16(fmt, dx.data_ptr(), dw.data_ptr(), out.data_ptr(), x.size, _stream())
    return out.cpu().numpy()


@pytest.mark.parametrize("fmt", [0, 1], ids=["e4m3", "e5m2"])
def test_sr16_encoder_at_threshold_draws_in_every_lane(fmt):
    """The hardware stochastic-rounding conversion (the encoder of 16-bit-draw
    stochastic rounding) against the oracle: the adversarial inputs of the
    32-bit encoder placed in each of the four codes of a word, each with the
    draw at its exact threshold, one below it, and a random one; the other
    three codes random values with random draws; a ragged last word."""
    rng = np.random.default_rng(61)
    xs, _, _ = pins.sr_cases(fmt, 31)
    live = np.isfinite(xs) & (np.abs(xs) < pins.FMAX[fmt])
    _, _, F = pins.sr16_threshold(fmt, np.where(live, xs, 0.0))
    T = 65536 - F
    draws = [np.clip(T, 0, 65535), np.clip(T - 1, 0, 65535), rng.integers(0, 1 << 16, xs.size)]
    for lane in range(4):
        for r in draws:
            r = r.astype(np.uint32)
            n = 4 * xs.size - 1  # ragged: the last word serves three codes
            x = (rng.standard_normal(4 * xs.size) * 10.0 ** rng.uniform(-8, 4, 4 * xs.size)).astype(np.float32)
            x[lane::4] = xs
            w = _sr16_words_for(r, np.full(xs.size, lane), rng)
            x = x[:n]
            got = _encode_sr16_device(fmt, x, w)
            exp = oracle.encode_sr16_words(fmt, x, w)
            d = np.flatnonzero(got != exp)
            assert d.size == 0, (lane, x[d[:8]], got[d[:8]], exp[d[:8]])


def test_sr16_encoder_edges():
    """n = 0 writes nothing; n = 1, 2, 3 write only their codes; invalid
    arguments are refused."""
    x = np.array([1.0625, -3.3, 1e-3], np.float32)
    w = np.array([0xFFFFFFFF], np.uint32)
    for fmt in (0, 1):
        for n in (1, 2, 3):
            dx = torch.from_numpy(x[:n].copy()).cuda()
            dw = torch.from_numpy(w.view(np.int32)).cuda()
            out = torch.full((4,), 0xAA, dtype=torch.uint8, device="cuda")
            capi.fp8adam_encode_sr16(fmt, dx.data_ptr(), dw.data_ptr(), out.data_ptr(), n, _stream())
            got = out.cpu().numpy()
            assert (got[:n] == oracle.encode_sr16_words(fmt, x[:n], w)).all()
            assert (got[n:] == 0xAA).all()
        out = torch.full((4,), 0xAA, dtype=torch.uint8, device="cuda")
        capi.fp8adam_encode_sr16(fmt, 0, 0, out.data_ptr(), 0, _stream())
        assert (out.cpu().numpy() == 0xAA).all()
    with pytest.raises(capi.Fp8AdamError) as e:
        capi.fp8adam_encode_sr16(2, 0, 0, 0, 1, _stream())
    assert e.value.code == capi.ERR_UNSUPPORTED_FMT
    with pytest.raises(capi.Fp8AdamError) as e:
        capi.fp8adam_encode_sr16(0, 0, 0, 0, 5, _stream())
    assert e.value.code == capi.ERR_INVALID_ARG


@pytest.mark.slow
@pytest.mark.parametrize("fmt", [0, 1], ids=["e4m3", "e5m2"])
def test_sr16_encoder_all_fp32_inputs(fmt):
    """Every fp32 bit pattern through the hardware stochastic-rounding
    conversion, each with a random 16-bit draw (random words, every lane),
    against the oracle's 16-bit-draw encoder (computed here in threads)."""
    from concurrent.futures import ThreadPoolExecutor
    import os
    chunk = 1 << 28
    out = torch.empty(chunk, dtype=torch.uint8, device="cuda")
    workers = max(1, min(32, os.cpu_count() or 1))
    part = chunk // 64
    bad = 0
    with ThreadPoolExecutor(workers) as pool:
        for first in range(0, 1 << 32, chunk):
            xh = np.arange(first, first + chunk, dtype=np.uint64).astype(np.uint32).view(np.float32)
            wh = np.random.default_rng(first // chunk + 100 * fmt).integers(
                0, 1 << 32, chunk // 4, dtype=np.uint64).astype(np.uint32)
            dx = torch.from_numpy(xh.view(np.int32)).cuda()
            dw = torch.from_numpy(wh.view(np.int32)).cuda()
            capi.fp8adam_encode_sr16(fmt, dx.data_ptr(), dw.data_ptr(), out.data_ptr(), chunk, _stream())
            got = out.cpu().numpy()
            del dx, dw
            exp = np.concatenate(list(pool.map(
                lambda s: oracle.encode_sr16_words(fmt, xh[s:s + part], wh[s // 4:(s + part) // 4]),
                range(0, chunk, part))))
            bad += int((got != exp).sum())
    assert bad == 0
