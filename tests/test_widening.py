"""The E4M3 -> bf16 widening the multi-token kernel applies to an E4M3 cache,
checked as arithmetic on the host for all 256 codes.

The kernel places a code's sign in bit 15 and its 7 exponent/mantissa bits in
bits 4..10 of a 16-bit word (byte permute with sign replication, shift by 4,
mask 0x87f0), reads the word as a bf16 and multiplies it by 2^120.  Here the
same bit operations run in NumPy, the bf16 word is read as a float exactly
(its bits padded to fp32), and the product is compared with the oracle's
decoding of the code: equal for every finite code, subnormals and both zeros
included, and +-480 for the two NaN codes (documented behaviour of that path).
"""

import numpy as np
import pytest

import oracle


def _widen(codes: np.ndarray) -> np.ndarray:
    c = codes.astype(np.uint32)
    sign_byte = np.where(c & 0x80, 0xFF, 0x00).astype(np.uint32)
    half = ((sign_byte << 8) | c) << 4                       # 16 bits of interest
    bf16_bits = (half & 0x87F0).astype(np.uint32)
    as_f32 = (bf16_bits << 16).view(np.float32).astype(np.float64)
    return as_f32 * 2.0 ** 120


def test_every_finite_code_widens_exactly():
    codes = np.arange(256, dtype=np.uint8)
    finite = (codes & 0x7F) != 0x7F
    got = _widen(codes[finite])
    want = oracle.e4m3_to_float(codes[finite]).astype(np.float64)
    assert np.array_equal(got, want)
    # signed zeros keep their sign
    assert np.signbit(_widen(np.array([0x80], dtype=np.uint8)))[0]
    assert not np.signbit(_widen(np.array([0x00], dtype=np.uint8)))[0]


def test_subnormal_codes_are_covered():
    sub = np.array([m for m in range(1, 8)] + [0x80 | m for m in range(1, 8)], dtype=np.uint8)
    got = _widen(sub)
    assert np.array_equal(np.abs(got[:7]), np.arange(1, 8) * 2.0 ** -9)
    assert np.array_equal(got[7:], -got[:7])


@pytest.mark.parametrize("code,value", [(0x7F, 480.0), (0xFF, -480.0)])
def test_nan_codes_read_as_480(code, value):
    assert np.isnan(oracle.e4m3_to_float(np.array([code], dtype=np.uint8)))[0]
    assert _widen(np.array([code], dtype=np.uint8))[0] == value
