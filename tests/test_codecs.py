"""Pins for the oracle's bf16 and E4M3 codecs.

The oracle's codecs are checked against things outside the oracle: numpy's
own binary32 reinterpretation, torch's float32->bf16 and float8_e4m3fn casts
(library routines), landmark values of the two formats stored under
tests/golden/, and exhaustive round trips and tie cases."""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_landmarks(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                code, value = line.split()
                rows.append((int(code, 16), float(value)))
    return rows


# ---- bf16 ------------------------------------------------------------------

def test_bf16_decode_all_patterns_match_binary32_reinterpretation():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = oracle.bf16_decode(bits)
    ref = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    # signed zeros survive
    assert math.copysign(1.0, got[0x8000]) == -1.0


def test_bf16_encode_roundtrips_every_non_nan_pattern():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = oracle.bf16_decode(bits)
    keep = ~np.isnan(vals)
    back = oracle.bf16_encode(vals[keep])
    assert np.array_equal(back, bits[keep])
    assert oracle.bf16_encode(np.array([np.nan]))[0] == 0x7FC0


def test_bf16_encode_ties_to_even_and_nearest_elsewhere():
    # all positive finite patterns whose successor is finite
    b = np.arange(0, 0x7F7F, dtype=np.uint16)
    lo = oracle.bf16_decode(b)
    hi = oracle.bf16_decode(b + 1)
    mid = (lo + hi) / 2.0                       # exact in fp64
    even = np.where(b % 2 == 0, b, b + 1).astype(np.uint16)
    assert np.array_equal(oracle.bf16_encode(mid), even)
    assert np.array_equal(oracle.bf16_encode(-mid), even | 0x8000)
    eps = (hi - lo) * 2.0 ** -20
    assert np.array_equal(oracle.bf16_encode(mid - eps), b)
    assert np.array_equal(oracle.bf16_encode(mid + eps), (b + 1).astype(np.uint16))


def test_bf16_encode_matches_torch_cast_of_float32_values():
    rng = np.random.default_rng(1)
    raw = rng.integers(0, 2 ** 32, size=200_000, dtype=np.uint64).astype(np.uint32)
    f32 = raw.view(np.float32)
    f32 = f32[np.isfinite(f32)]
    # torch rounds float32 -> bf16 to nearest even (a single rounding)
    ref = torch.from_numpy(f32.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.bf16_encode(f32.astype(np.float64))
    assert np.array_equal(got, ref)


def test_bf16_overflow_and_landmarks():
    assert oracle.bf16_encode(np.array([3.5e38]))[0] == 0x7F80          # rounds past max
    assert oracle.bf16_encode(np.array([-np.inf]))[0] == 0xFF80
    for code, value in _read_landmarks("bf16_landmarks.txt"):
        assert oracle.bf16_decode(np.array([code], np.uint16))[0] == value
        assert oracle.bf16_encode(np.array([value]))[0] == code


# ---- E4M3 ------------------------------------------------------------------

def test_e4m3_decode_all_codes_match_torch_float8():
    codes = np.arange(256, dtype=np.uint8)
    got = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    nan = np.isnan(ref)
    assert set(np.nonzero(nan)[0]) == {0x7F, 0xFF}
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_e4m3_landmarks_from_the_format_definition():
    for code, value in _read_landmarks("e4m3_landmarks.txt"):
        assert oracle.e4m3_decode(np.array([code], np.uint8))[0] == value
        assert oracle.e4m3_encode(np.array([value], np.float32))[0] == code


def test_e4m3_encode_roundtrip_ties_and_saturation():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    vals = oracle.e4m3_decode(codes)
    back = oracle.e4m3_encode(vals.astype(np.float32))
    assert np.array_equal(back, codes)
    # midpoints between neighbours tie to the even code
    pos = np.arange(0, 0x7E, dtype=np.uint8)
    lo, hi = oracle.e4m3_decode(pos), oracle.e4m3_decode(pos + 1)
    mid = ((lo + hi) / 2).astype(np.float32)            # exact in fp32
    even = np.where(pos % 2 == 0, pos, pos + 1).astype(np.uint8)
    assert np.array_equal(oracle.e4m3_encode(mid), even)
    assert np.array_equal(oracle.e4m3_encode(-mid), even | 0x80)
    # saturation to +-448, NaN stays NaN
    sat = np.array([448, 449, 464, 465, 1e6, np.inf, -500, -np.inf], np.float32)
    assert list(oracle.e4m3_encode(sat)) == [0x7E] * 6 + [0xFE] * 2
    assert oracle.e4m3_encode(np.array([np.nan], np.float32))[0] == 0x7F


def test_e4m3_encode_matches_torch_cast_where_torch_is_finite():
    rng = np.random.default_rng(2)
    x = np.concatenate([
        rng.standard_normal(200_000) * 100,
        rng.standard_normal(50_000) * 2.0 ** -7,         # subnormal range
        rng.uniform(-463.9, 463.9, 50_000),
    ]).astype(np.float32)
    # torch's cast rounds to nearest even and turns overflow into NaN; inside
    # |x| < 464 it never overflows, so there it is the same function
    x = x[np.abs(x) < 464]
    ref = torch.from_numpy(x.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(x)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("v", [2.0 ** -10, 3 * 2.0 ** -11, 2.0 ** -9 * 1.5, 2.0 ** -6 * (1 - 1 / 16)])
def test_e4m3_subnormal_rounding(v):
    ref = torch.tensor([v], dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).item()
    assert oracle.e4m3_encode(np.array([v], np.float32))[0] == ref
