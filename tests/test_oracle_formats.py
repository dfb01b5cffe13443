"""Pins for the oracle's E2M1 / E4M3 / E8M0 codecs against library codecs and spec tables."""
import math

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle.formats import (E2M1_MAGNITUDES, E4M3_MAGNITUDES, e2m1_decode, e2m1_encode,
                            e4m3_decode, e4m3_encode, e8m0_decode)
from tests.golden_io import load


def test_e2m1_table_matches_ocp_spec():
    g = load("e2m1_table.txt")
    got = e2m1_decode(np.array(g["codes"], dtype=np.uint8))
    want = np.array(g["values"], dtype=np.float64)
    assert np.array_equal(got, want)
    # sign of zero: code 8 is negative zero
    assert math.copysign(1.0, got[8]) == -1.0 and math.copysign(1.0, got[0]) == 1.0


def test_e2m1_decode_matches_ml_dtypes_all_codes():
    lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    ours = e2m1_decode(np.arange(16, dtype=np.uint8))
    assert np.array_equal(np.signbit(lib), np.signbit(ours))
    assert np.array_equal(lib, ours)


def _sweep(lo, hi, n, rng, table):
    """Random float32 values in [lo, hi], every midpoint of ``table`` and its two fp32 neighbours."""
    v = rng.uniform(lo, hi, size=n).astype(np.float32)
    mids = ((table[1:] + table[:-1]) / 2).astype(np.float32)
    extra = np.concatenate([mids, np.nextafter(mids, np.float32(np.inf)),
                            np.nextafter(mids, np.float32(0)), table.astype(np.float32)])
    v = np.concatenate([v, extra, -extra, -v])
    return v


def test_e2m1_encode_matches_ml_dtypes_rne_satfinite():
    rng = np.random.default_rng(0)
    v = _sweep(0, 8, 200_000, rng, E2M1_MAGNITUDES)
    v = np.concatenate([v, np.float32([1e6, -1e6, 6.5, -7.0, 1e-30, -1e-30, 0.0, -0.0])])
    lib = v.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    assert np.array_equal(e2m1_encode(v), lib)


def test_e2m1_midpoints_round_to_even_code():
    # midpoints between neighbours go to the code with a 0 low bit
    mids = np.float32([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    assert list(e2m1_encode(mids)) == [0, 2, 2, 4, 4, 6, 6]
    assert list(e2m1_encode(-mids)) == [8, 10, 10, 12, 12, 14, 14]


def test_e2m1_roundtrip_all_codes():
    codes = np.arange(16, dtype=np.uint8)
    assert np.array_equal(e2m1_encode(e2m1_decode(codes).astype(np.float32)), codes)


def test_e4m3_decode_matches_torch_all_codes():
    lib = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    ours = e4m3_decode(np.arange(256, dtype=np.uint8))
    assert np.array_equal(np.isnan(lib), np.isnan(ours))
    ok = ~np.isnan(lib)
    assert np.array_equal(lib[ok], ours[ok])
    assert np.array_equal(np.signbit(lib[ok]), np.signbit(ours[ok]))


def test_e4m3_points_match_ocp_spec():
    g = load("e4m3_points.txt")
    assert np.array_equal(e4m3_decode(np.array(g["codes"], dtype=np.uint8)), np.array(g["values"], float))
    assert np.all(np.isnan(e4m3_decode(np.array(g["nan_codes"], dtype=np.uint8))))


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(1)
    a = _sweep(0, 460, 200_000, rng, E4M3_MAGNITUDES)
    b = _sweep(0, 2.0 ** -5, 100_000, rng, E4M3_MAGNITUDES[E4M3_MAGNITUDES < 2.0 ** -5])
    v = np.concatenate([a, b])
    v = v[np.abs(v) < 464]  # torch turns values past the 448/480 midpoint into NaN (no saturation)
    lib = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(e4m3_encode(v), lib)


def test_e4m3_encode_saturates():
    v = np.float32([448, 450, 463.9, 464, 500, 1e9, 3e38])
    assert np.all(e4m3_encode(v) == 0x7E)
    assert np.all(e4m3_encode(-v) == 0xFE)


def test_e8m0_decode_matches_torch_all_codes():
    lib = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e8m0fnu).double().numpy()
    ours = e8m0_decode(np.arange(256))
    assert np.array_equal(np.isnan(lib), np.isnan(ours))
    ok = ~np.isnan(lib)
    assert np.array_equal(lib[ok], ours[ok])


@pytest.mark.parametrize("code", [0, 1, 126, 127, 128, 254])
def test_e8m0_closed_form(code):
    assert e8m0_decode(np.array([code]))[0] == math.ldexp(1.0, code - 127)
