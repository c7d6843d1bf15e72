"""Pins for the oracle's hand-written IEEE binary16 conversions.

The library routine numpy ``float32.astype(float16)`` (round to nearest even)
is the independent reference; the sets below are chosen so that every rounding
class of every exponent is reached: all sign/exponent/upper-fraction patterns
with the dropped bits at and around the halfway point, the full fraction range
of every exponent whose result is a binary16 subnormal, and a large stride of
the whole 2^32 space.  Setting Q4_EXHAUSTIVE=1 runs every one of the 2^32
patterns (several minutes).
"""
import os

import numpy as np
import pytest

import oracle


def _check(bits_u32: np.ndarray):
    f = bits_u32.view(np.float32)
    with np.errstate(over="ignore"):
        want = f.astype(np.float16).view(np.uint16)
    got = oracle.f32_to_f16_bits(f)
    nan = np.isnan(f)
    # NaN payloads are not specified; only NaN-ness and the sign are compared.
    assert np.array_equal(got[~nan], want[~nan])
    g = got[nan]
    assert np.all((g & 0x7C00) == 0x7C00) and np.all((g & 0x3FF) != 0)
    assert np.array_equal(g >> 15, (bits_u32[nan] >> 31).astype(np.uint16))


def test_named_values():
    cases = [
        (0.0, 0x0000), (-0.0, 0x8000), (1.0, 0x3C00), (-2.0, 0xC000), (0.1, 0x2E66), (1 / 3, 0x3555),
        (65504.0, 0x7BFF), (65519.99, 0x7BFF), (65520.0, 0x7C00), (1e6, 0x7C00), (2.0 ** -24, 0x0001),
        (2.0 ** -25, 0x0000), (1.5 * 2.0 ** -25, 0x0001), (2.0 ** -14, 0x0400), (0.25, 0x3400),
        (float("inf"), 0x7C00), (float("-inf"), 0xFC00),
    ]
    for v, h in cases:
        assert int(oracle.f32_to_f16_bits(np.float32(v)).reshape(-1)[0]) == h, v


def test_rounding_classes_all_exponents():
    hi = np.arange(1 << 19, dtype=np.uint32) << 13          # sign, exponent, top 10 fraction bits
    for low in (0, 1, 0x0FFF, 0x1000, 0x1001, 0x1FFF):
        _check(hi | np.uint32(low))


def test_subnormal_results_full_fraction():
    frac = np.arange(1 << 23, dtype=np.uint32)
    for e in range(-26, -13):                              # results below the binary16 normal range
        for sign in (0, 1):
            _check((np.uint32(sign) << 31) | (np.uint32(e + 127) << 23) | frac)


def test_strided_space():
    _check(np.arange(0, 1 << 32, 251, dtype=np.uint64).astype(np.uint32))


@pytest.mark.skipif(os.environ.get("Q4_EXHAUSTIVE") != "1", reason="set Q4_EXHAUSTIVE=1 for all 2^32 inputs")
def test_exhaustive():
    step = 1 << 24
    for start in range(0, 1 << 32, step):
        _check(np.arange(start, start + step, dtype=np.uint64).astype(np.uint32))


def test_f16_to_f32_all_patterns():
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = oracle.f16_bits_to_f32(h)
    want = h.view(np.float16).astype(np.float32)
    nan = np.isnan(want)
    assert np.array_equal(got[~nan].view(np.uint32), want[~nan].view(np.uint32))
    assert np.all(np.isnan(got[nan]))
    # and back: every non-NaN binary16 value survives the round trip
    back = oracle.f32_to_f16_bits(got)
    assert np.array_equal(back[~nan], h[~nan])
