"""Pins for the oracle's storage decoders and its E4M3 encoder.

Every decoder is checked over all codes against an independent library
conversion (numpy float16, torch bfloat16 / float8_e4m3fn) and against closed
forms of the formats; the encoder against torch's round-to-nearest-even
conversion inside the range, every midpoint (ties to even) and saturation.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def _same(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return np.array_equal(np.isnan(a), np.isnan(b)) and np.array_equal(
        np.nan_to_num(a, nan=0.0), np.nan_to_num(b, nan=0.0))


def test_f16_all_codes_match_numpy():
    codes = np.arange(1 << 16, dtype=np.uint16)
    got = oracle.values(codes, "f16")
    ref = codes.view(np.float16).astype(np.float64)
    assert _same(got, ref)


def test_bf16_all_codes_match_torch():
    codes = np.arange(1 << 16, dtype=np.uint16)
    got = oracle.values(codes, "bf16")
    ref = torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert _same(got, ref)


def test_f32_random_codes_match_numpy():
    rng = np.random.default_rng(7)
    codes = rng.integers(0, 1 << 32, size=200000, dtype=np.uint64).astype(np.uint32)
    got = oracle.values(codes, "f32")
    assert _same(got, codes.view(np.float32).astype(np.float64))


def test_e4m3_all_codes_match_torch_and_closed_forms():
    codes = np.arange(256, dtype=np.uint8)
    got = oracle.values(codes, "fp8_e4m3")
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert _same(got, ref)
    # closed forms of the OCP E4M3 format
    assert got[0x7E] == 448.0 and got[0xFE] == -448.0          # 1.75 * 2^8, largest finite
    assert got[0x01] == 2.0 ** -9                               # smallest subnormal
    assert got[0x07] == 7 * 2.0 ** -9                           # largest subnormal
    assert got[0x08] == 2.0 ** -6                               # smallest normal
    assert got[0x38] == 1.0                                     # exponent field 7 = bias
    assert math.isnan(got[0x7F]) and math.isnan(got[0xFF])      # S.1111.111
    assert got[0x80] == 0.0 and math.copysign(1, got[0x80]) < 0
    assert np.isfinite(got[np.r_[0:0x7F, 0x80:0xFF]]).all()     # no infinities
    pos = got[:0x7F]
    assert np.all(np.diff(pos) > 0)                             # monotone in the code


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.normal(0, 1, 100000), rng.normal(0, 100, 100000),
                        rng.uniform(-448, 448, 50000), rng.normal(0, 0.01, 50000)])
    x = np.clip(x, -448, 448).astype(np.float32)   # torch turns out-of-range values into NaN
    got = oracle.e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)


def test_e4m3_encode_midpoints_tie_to_even():
    vals = oracle.values(np.arange(0x7F, dtype=np.uint8), "fp8_e4m3")
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (vals[:-1] + vals[1:]) / 2)  # exact in f32
    got = oracle.e4m3_encode(mids)
    lo = np.arange(0x7E, dtype=np.uint8)
    expect = np.where(lo % 2 == 0, lo, lo + 1).astype(np.uint8)
    assert np.array_equal(got, expect)
    assert np.array_equal(oracle.e4m3_encode(-mids), expect | 0x80)
    # a hair either side of every midpoint goes to the nearer code
    up = np.nextafter(mids, np.float32(np.inf))
    dn = np.nextafter(mids, np.float32(-np.inf))
    assert np.array_equal(oracle.e4m3_encode(up), lo + 1)
    assert np.array_equal(oracle.e4m3_encode(dn), lo)


def test_e4m3_encode_saturates_and_nan():
    big = np.array([448.0, 449.0, 463.99, 464.0, 465.0, 1e6, np.inf], dtype=np.float32)
    assert (oracle.e4m3_encode(big) == 0x7E).all()
    assert (oracle.e4m3_encode(-big) == 0xFE).all()
    assert oracle.e4m3_encode(np.array([np.nan], np.float32))[0] == 0x7F
    assert oracle.e4m3_encode(np.array([0.0], np.float32))[0] == 0x00
    assert oracle.e4m3_encode(np.array([-0.0], np.float32))[0] == 0x80
    # below half the smallest subnormal -> 0; exactly half -> tie to even code 0
    assert oracle.e4m3_encode(np.array([2.0 ** -10], np.float32))[0] == 0x00
    assert oracle.e4m3_encode(np.array([1.5 * 2.0 ** -9], np.float32))[0] == 0x02
