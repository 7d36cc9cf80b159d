"""Pins for the oracle's e4m3 encoder and per-token FP8 quantiser (CPU only).

The encoder is checked against the format itself (every finite code round-trips, midpoints
between neighbouring values go to the even code, saturation, NaN, signed zero) and against an
independent implementation (torch's float8_e4m3fn cast, which rounds to nearest even); the
quantiser against its per-row rule and the e4m3 error bound.
"""

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def test_every_finite_code_round_trips():
    codes = np.arange(256, dtype=np.uint8)
    vals = oracle.decode_e4m3(codes)
    finite = ~np.isnan(vals)
    assert np.array_equal(oracle.encode_e4m3(vals[finite]), codes[finite])


def test_midpoints_round_to_even_code():
    pos = oracle.decode_e4m3(np.arange(127, dtype=np.uint8))
    mids = (pos[:-1] + pos[1:]) / 2.0
    got = oracle.encode_e4m3(mids)
    lo = np.arange(126)
    want = np.where(lo % 2 == 0, lo, lo + 1)
    assert np.array_equal(got, want.astype(np.uint8))
    # just off the midpoint goes to the nearer neighbour
    eps = (pos[1:] - pos[:-1]) * 1e-3
    assert np.array_equal(oracle.encode_e4m3(mids - eps), lo.astype(np.uint8))
    assert np.array_equal(oracle.encode_e4m3(mids + eps), (lo + 1).astype(np.uint8))


def test_saturation_nan_and_signed_zero():
    y = np.array([448.0, 448.5, 464.0, 1e9, np.inf, -448.0, -1e9, -np.inf, np.nan, 0.0, -0.0, -1e-30])
    got = oracle.encode_e4m3(y)
    assert list(got) == [126, 126, 126, 126, 126, 254, 254, 254, 0x7F, 0x00, 0x80, 0x80]


def test_agrees_with_torch_cast():
    rng = np.random.default_rng(5)
    y = np.concatenate([rng.standard_normal(100000) * 50, rng.standard_normal(20000) * 1e-3,
                        rng.uniform(-448, 448, 20000)]).astype(np.float32)
    ref = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.encode_e4m3(y), ref)


def test_quantiser_row_rule_and_error_bound():
    rng = np.random.default_rng(7)
    x = torch.from_numpy(rng.standard_normal((40, 256)).astype(np.float32) * rng.uniform(1e-3, 1e3, (40, 1))
                         ).to(torch.bfloat16).float().numpy()
    x[3] = 0.0                                   # all-zero row: scale 1, codes 0
    x[5, 17] = np.nan                            # NaN takes no part in the maximum
    codes, scale = oracle.quantize_fp8_rows(x)
    assert scale.dtype == np.float32 and scale[3] == 1.0 and not codes[3].any()
    assert codes[5, 17] in (0x7F, 0xFF)
    amax = np.nanmax(np.abs(x), axis=1).astype(np.float32)
    rows = np.arange(40) != 3
    assert np.array_equal(scale[rows], (amax[rows] / np.float32(448)).astype(np.float32))
    # the largest element lands on the largest code (exact quotient or saturated)
    assert np.all(np.abs(oracle.decode_e4m3(codes[rows]))[np.arange(40)[rows] != 5].max(axis=1) == 448.0)
    # relative error of a normal e4m3 code is at most 2^-4 of the value; absolute at most
    # half the subnormal step (2^-10) times the scale below the normal range
    deq = oracle.decode_e4m3(codes) * scale[:, None].astype(np.float64)
    ok = ~np.isnan(x)
    err = np.abs(deq - x)[ok]
    bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * np.broadcast_to(scale[:, None], x.shape))[ok]
    assert np.all(err <= bound * (1 + 1e-6))
