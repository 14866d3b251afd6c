"""Pins for the oracle's E4M3 codec against facts fixed outside the oracle.

E4M3 is the FP8 format of every operand ("DeepSeek-V3 Technical Report" summary page, Key ideas,
FP8 mixed-precision bullet).  The pages name the format only; the OCP E4M3FN definition (bias 7,
largest finite 448, NaN at S.1111.111, subnormals m * 2^-9), round-to-nearest-even and saturation
to 448 are this library's reading.  Pins:

* closed-form values of specific codes;
* exhaustive decode -> encode round trip over all 256 codes;
* every tie between adjacent codes goes to the even code, one binary32 ulp off the tie goes to
  the nearer code;
* saturation of finite values above 448;
* a library cross-check against PyTorch's float8_e4m3fn cast on 2^20 random in-range values and
  on every tie and near-tie.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def test_closed_form_values():
    dec = oracle.e4m3_decode(np.arange(256, dtype=np.uint8))
    assert dec[0x7E] == 448.0
    assert dec[0xFE] == -448.0
    assert dec[0x08] == 2.0 ** -6          # smallest normal
    assert dec[0x01] == 2.0 ** -9          # smallest subnormal
    assert dec[0x07] == 7 * 2.0 ** -9      # largest subnormal
    assert dec[0x38] == 1.0                # exponent field 7 = bias
    assert dec[0x3C] == 1.5
    assert dec[0x77] == 240.0
    assert dec[0x00] == 0.0 and not math.copysign(1.0, dec[0x00]) < 0
    assert dec[0x80] == 0.0 and math.copysign(1.0, dec[0x80]) < 0
    assert math.isnan(dec[0x7F]) and math.isnan(dec[0xFF])
    pos = dec[:0x7F]
    assert np.all(np.diff(pos) > 0), "positive codes must decode in increasing order"
    assert np.all(dec[0x80:0xFF] == -pos)


def test_roundtrip_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    dec = oracle.e4m3_decode(codes)
    finite = ~np.isnan(dec)
    back = oracle.e4m3_encode(dec[finite].astype(np.float32))
    assert np.array_equal(back, codes[finite])
    # NaN encodes to NaN codes with the sign kept.
    assert oracle.e4m3_encode(np.float32(np.nan))[()] & 0x7F == 0x7F


def _ties():
    dec = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    lo = dec[:-1]
    hi = dec[1:]
    mid = ((lo + hi) / 2).astype(np.float32)
    assert np.all(mid.astype(np.float64) == (lo + hi) / 2), "ties are exact in binary32"
    return np.arange(0x7E, dtype=np.uint8), mid


def test_ties_to_even_and_neighbours():
    c, mid = _ties()
    even = np.where(c % 2 == 0, c, c + 1).astype(np.uint8)
    assert np.array_equal(oracle.e4m3_encode(mid), even)
    up = np.nextafter(mid, np.float32(np.inf))
    down = np.nextafter(mid, np.float32(0))
    assert np.array_equal(oracle.e4m3_encode(up), (c + 1).astype(np.uint8))
    assert np.array_equal(oracle.e4m3_encode(down), c)
    # Negative side mirrors with the sign bit.
    assert np.array_equal(oracle.e4m3_encode(-mid), even | 0x80)
    assert np.array_equal(oracle.e4m3_encode(-up), (c + 1).astype(np.uint8) | 0x80)


def test_saturation_and_tiny():
    big = np.array([448.0, 449.0, 463.99, 464.0, 470.0, 480.0, 1e6, 1e30, np.inf],
                   dtype=np.float32)
    assert np.all(oracle.e4m3_encode(big) == 0x7E)
    assert np.all(oracle.e4m3_encode(-big) == 0xFE)
    tiny = np.array([0.0, 1e-40, 2.0 ** -11, 2.0 ** -10], dtype=np.float32)
    assert np.all(oracle.e4m3_encode(tiny) == 0x00)     # 2^-10 is the tie 0 | 2^-9: even is 0
    assert np.all(oracle.e4m3_encode(-tiny) == 0x80)    # sign of zero kept
    assert oracle.e4m3_encode(np.float32(np.nextafter(np.float32(2.0 ** -10), np.float32(1))))[()] == 0x01


def _torch_codes(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_cross_check_torch_random():
    g = np.random.Generator(np.random.PCG64(1234))
    # Log-uniform magnitudes over the whole E4M3 range and below, random signs.
    mag = np.exp2(g.uniform(-14.0, math.log2(448.0), size=1 << 20)).astype(np.float32)
    mag = np.minimum(mag, np.float32(448.0))
    x = np.where(g.random(mag.size) < 0.5, -mag, mag).astype(np.float32)
    assert np.array_equal(oracle.e4m3_encode(x), _torch_codes(x))


def test_cross_check_torch_ties():
    _, mid = _ties()
    pts = np.concatenate([mid, np.nextafter(mid, np.float32(np.inf)),
                          np.nextafter(mid, np.float32(0))])
    pts = np.concatenate([pts, -pts])
    assert np.array_equal(oracle.e4m3_encode(pts), _torch_codes(pts))


def test_exhaustive_binary32_against_torch():
    """Every binary32 bit pattern with |x| <= 464 (both signs, zeros, subnormals): the oracle's
    encoder agrees with PyTorch's float8_e4m3fn cast.  Up to 464 the nearest-even rounding of
    either encoder never needs saturation (464 is the tie between 448 and the first value past
    the E4M3 range, and it rounds to the even code 448), so the two must be identical."""
    top = int(np.array([464.0], dtype=np.float32).view(np.uint32)[0])   # 0x43E80000
    chunk = 1 << 24
    for sign in (0, 0x80000000):
        for lo in range(0, top + 1, chunk):
            bits = np.arange(lo, min(lo + chunk, top + 1), dtype=np.uint32) | np.uint32(sign)
            x = bits.view(np.float32)
            got, want = oracle.e4m3_encode(x), _torch_codes(x)
            if not np.array_equal(got, want):
                i = int(np.flatnonzero(got != want)[0])
                raise AssertionError(f"pattern {bits[i]:#010x} ({x[i]!r}): oracle {got[i]:#04x}, "
                                     f"torch {want[i]:#04x}")
