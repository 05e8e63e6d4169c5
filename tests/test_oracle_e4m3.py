"""Pins for the oracle's E4M3 decoder and encoder.

The oracle's encoder is written from the OCP FP8 E4M3 format (bias 7, 3 mantissa
bits, largest finite 448, S.1111.111 NaN, no infinities) with round-to-nearest-even
and saturation at 448.  These tests pin it to things other than itself:

* the value of every code against torch's independent ``float8_e4m3fn`` decoder;
* the round trip code -> value -> code for all 254 non-NaN codes;
* every decision boundary (each midpoint between neighbouring grid values and the
  floats on either side of it), checked against the ties-to-even rule;
* a large random sample against a nearest-grid-point search written here with
  numpy (a search over the grid, not the encoder's exponent/mantissa arithmetic);
* in-range values against torch's independent fp32 -> e4m3fn conversion.
"""
import numpy as np
import pytest
import torch

import oracle

ALL_CODES = np.arange(256, dtype=np.uint8)
NAN_CODES = {0x7F, 0xFF}
FINITE = np.array([c for c in range(256) if c not in NAN_CODES], dtype=np.uint8)


def torch_decode(codes: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def test_value_of_every_code_matches_torch():
    v = oracle.e4m3_value(ALL_CODES)
    ref = torch_decode(ALL_CODES)
    for c in range(256):
        if c in NAN_CODES:
            assert np.isnan(v[c])
        else:
            assert v[c] == ref[c], hex(c)
            assert np.signbit(v[c]) == bool(c & 0x80), hex(c)


def test_format_landmarks():
    v = oracle.e4m3_value(np.array([0x7E, 0xFE, 0x01, 0x07, 0x08, 0x38, 0x00, 0x80], np.uint8))
    assert list(v[:6]) == [448.0, -448.0, 2.0 ** -9, 7 * 2.0 ** -9, 2.0 ** -6, 1.0]
    assert v[6] == 0.0 and not np.signbit(v[6])
    assert v[7] == 0.0 and np.signbit(v[7])


def test_round_trip_all_finite_codes():
    vals = oracle.e4m3_value(FINITE).astype(np.float32)
    assert np.array_equal(oracle.e4m3_encode(vals), FINITE)


def _positive_grid():
    codes = np.arange(0x00, 0x7F, dtype=np.uint8)  # 0 .. 0x7E, increasing values
    vals = oracle.e4m3_value(codes)
    assert np.all(np.diff(vals) > 0)
    return codes, vals


def test_every_midpoint_and_its_neighbours():
    codes, vals = _positive_grid()
    lo, hi = vals[:-1], vals[1:]
    mid = ((lo + hi) / 2).astype(np.float32)
    assert np.array_equal(mid.astype(np.float64), (lo + hi) / 2)  # midpoints are exact in fp32
    even = np.where(codes[:-1] % 2 == 0, codes[:-1], codes[1:])
    below = np.nextafter(mid, np.float32(0))
    above = np.nextafter(mid, np.float32(np.inf))
    for sign in (1.0, -1.0):
        sbit = 0x80 if sign < 0 else 0
        assert np.array_equal(oracle.e4m3_encode(sign * mid), even | sbit)
        assert np.array_equal(oracle.e4m3_encode(sign * below), codes[:-1] | sbit)
        assert np.array_equal(oracle.e4m3_encode(sign * above), codes[1:] | sbit)


def test_saturation_and_zeros():
    big = np.array([448.0, np.nextafter(np.float32(448), np.float32(1e9)), 463.99997, 464.0,
                    480.0, 1e10, 3.4e38], dtype=np.float32)
    assert np.all(oracle.e4m3_encode(big) == 0x7E)
    assert np.all(oracle.e4m3_encode(-big) == 0xFE)
    z = oracle.e4m3_encode(np.array([0.0, -0.0, 1e-30, -1e-30, 2.0 ** -10, -(2.0 ** -10)],
                                    dtype=np.float32))
    assert list(z) == [0x00, 0x80, 0x00, 0x80, 0x00, 0x80]


def nearest_grid_search(t: np.ndarray) -> np.ndarray:
    """Nearest E4M3 code by searching the grid; ties to the even code; saturate."""
    codes, vals = _positive_grid()
    a = np.abs(t.astype(np.float64))
    idx = np.clip(np.searchsorted(vals, a), 1, len(vals) - 1)
    lo, hi = vals[idx - 1], vals[idx]
    dlo, dhi = a - lo, hi - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (codes[idx] % 2 == 0))
    out = np.where(pick_hi, codes[idx], codes[idx - 1]).astype(np.uint8)
    out = np.where(a >= vals[-1], np.uint8(0x7E), out)
    out = np.where(a <= 0, np.uint8(0), out)
    return out | np.where(np.signbit(t), np.uint8(0x80), np.uint8(0))


@pytest.mark.parametrize("seed", [0, 1])
def test_random_bit_patterns_against_grid_search(seed):
    rng = np.random.default_rng(seed)
    bits = rng.integers(0, 2 ** 32, size=1 << 20, dtype=np.uint64).astype(np.uint32)
    t = bits.view(np.float32)
    t = t[np.isfinite(t)]
    assert np.array_equal(oracle.e4m3_encode(t), nearest_grid_search(t))


@pytest.mark.parametrize("seed", [2, 3])
def test_dense_range_against_grid_search(seed):
    # magnitudes spread log-uniformly over the whole E4M3 range and a bit beyond
    rng = np.random.default_rng(seed)
    mag = np.exp2(rng.uniform(-14, 9.2, size=1 << 20)).astype(np.float32)
    t = np.where(rng.random(mag.size) < 0.5, -mag, mag).astype(np.float32)
    assert np.array_equal(oracle.e4m3_encode(t), nearest_grid_search(t))


def test_in_range_values_against_torch_conversion():
    rng = np.random.default_rng(4)
    mag = np.exp2(rng.uniform(-14, np.log2(448.0), size=1 << 20)).astype(np.float32)
    t = np.where(rng.random(mag.size) < 0.5, -mag, mag).astype(np.float32)
    t = np.concatenate([t, oracle.e4m3_value(FINITE).astype(np.float32)])
    ref = torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(t), ref)
