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
