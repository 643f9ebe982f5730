"""Pins for the oracle's e4m3 codec (CPU only).

The codec is written from the OCP FP8 E4M3 bit layout; here it is checked
against two independent implementations (ml_dtypes and torch's
float8_e4m3fn) and against values fixed by the format definition.
"""

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import e4m3


def test_decode_exhaustive_matches_two_libraries():
    codes = np.arange(256, dtype=np.uint8)
    ours = e4m3.decode(codes)
    ml = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    th = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ours)
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]
    assert np.array_equal(np.isnan(ml), nan) and np.array_equal(np.isnan(th), nan)
    assert np.array_equal(ours[~nan], ml[~nan])
    assert np.array_equal(ours[~nan], th[~nan])
    # signed zeros
    assert np.signbit(ours[0x80]) and not np.signbit(ours[0x00])


@pytest.mark.parametrize("value,code", [
    (0.0, 0x00), (-0.0, 0x80), (1.0, 0x38), (-1.0, 0xB8), (448.0, 0x7E), (-448.0, 0xFE),
    (2.0 ** -9, 0x01), (2.0 ** -6, 0x08), (7 * 2.0 ** -9, 0x07), (1.75, 0x3E), (240.0, 0x77),
    (256.0, 0x78), (0.5, 0x30),
])
def test_definition_values(value, code):
    assert e4m3.encode_rn_sat(np.float32(value)) == code
    d = e4m3.decode(np.uint8(code))
    assert d == value and np.signbit(d) == np.signbit(value)


def test_roundtrip_all_finite_codes():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    assert np.array_equal(e4m3.encode_rn_sat(e4m3.decode(codes)), codes)


def test_grid_monotone():
    pos = e4m3.decode(np.arange(0x7F, dtype=np.uint8))
    assert np.all(np.diff(pos) > 0)


def test_midpoints_tie_to_even_code():
    pos = e4m3.decode(np.arange(0x7F, dtype=np.uint8))
    mids = (pos[:-1] + pos[1:]) / 2  # exactly representable in float32
    got = e4m3.encode_rn_sat(mids.astype(np.float32))
    lo = np.arange(0x7E)
    want = np.where(lo % 2 == 0, lo, lo + 1)
    assert np.array_equal(got, want)
    got_neg = e4m3.encode_rn_sat(-mids.astype(np.float32))
    assert np.array_equal(got_neg, want | 0x80)


def test_saturation():
    big = np.array([448.0, 448.0001, 463.9, 464.0, 480.0, 1e6, 3.0e38], dtype=np.float32)
    assert np.all(e4m3.encode_rn_sat(big) == 0x7E)
    assert np.all(e4m3.encode_rn_sat(-big) == 0xFE)


def test_tiny_values_round_to_signed_zero():
    assert e4m3.encode_rn_sat(np.float32(2.0 ** -10)) == 0x00  # tie between 0 and 2^-9 -> even (0)
    assert e4m3.encode_rn_sat(np.float32(-2.0 ** -10)) == 0x80
    assert e4m3.encode_rn_sat(np.float32(3 * 2.0 ** -11)) == 0x01  # 0.75 * 2^-9 -> 2^-9
    assert e4m3.encode_rn_sat(np.float32(-1e-30)) == 0x80


def test_random_against_library_casts_in_range():
    rng = np.random.default_rng(1234)
    # log-uniform magnitudes over the whole finite range and below it, both signs
    mag = np.exp2(rng.uniform(-14, np.log2(460.0), size=400_000)).astype(np.float32)
    v = np.where(rng.integers(0, 2, size=mag.size) == 1, -mag, mag).astype(np.float32)
    ours = e4m3.encode_rn_sat(v)
    ml = v.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    th = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ml)
    assert np.array_equal(ours, th)


def test_all_float32_midpoint_neighbours():
    """One float32 ulp either side of every midpoint must round away from the tie."""
    pos = e4m3.decode(np.arange(0x7F, dtype=np.uint8))
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    below = np.nextafter(mids, np.float32(0))
    above = np.nextafter(mids, np.float32(np.inf))
    assert np.array_equal(e4m3.encode_rn_sat(below), np.arange(0x7E))
    assert np.array_equal(e4m3.encode_rn_sat(above), np.arange(1, 0x7F))
