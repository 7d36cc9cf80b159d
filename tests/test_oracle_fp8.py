"""Pins for the oracle's e4m3 decoder: every code against an independent library decoder."""
import numpy as np
import torch

import oracle


def test_all_codes_match_library_decoder():
    codes = torch.arange(256, dtype=torch.uint8)
    lib = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = oracle.decode_e4m3(np.arange(256))
    nan_lib = np.isnan(lib)
    assert np.array_equal(nan_lib, np.isnan(ours))
    assert np.array_equal(lib[~nan_lib], ours[~nan_lib])


def test_hand_checked_code_points():
    t = oracle.e4m3_table()
    assert t[0x7E] == 448.0 and t[0xFE] == -448.0          # largest finite
    assert t[0x01] == 2.0 ** -9                              # smallest subnormal
    assert t[0x08] == 2.0 ** -6                              # smallest normal
    assert t[0x38] == 1.0 and t[0xB8] == -1.0
    assert t[0x00] == 0.0 and np.signbit(t[0x80])            # +0 and -0
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])           # the only NaNs, no infinities
    assert np.isfinite(t[np.r_[0:0x7F, 0x80:0xFF]]).all()


def test_every_finite_code_is_integer_multiple_of_2_pow_minus_9():
    t = oracle.e4m3_table()
    fin = t[np.isfinite(t)]
    n = fin * 2.0 ** 9
    assert np.array_equal(n, np.round(n)) and np.abs(n).max() == 448 * 512
