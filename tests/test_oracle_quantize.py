"""Pins for the oracle quantiser (4-bit symmetric, group 32, binary16 scale).

Checked against: hand-derived encodings (tests/golden/quantize_cases.json),
exact reconstruction of weights already on the integer grid, the per-element
round-trip bound |w - w'| <= s/2, an independent binary64 characterisation of
the code as the nearest integer in [-8, 7] (ties to even), the scale as the
binary16 cast of f32(amax)/7 through numpy's own conversion, the structural
facts every encoded group must satisfy, and (hypothesis) the same scale and
nearest-integer rules on arbitrary finite float32 groups spanning every binade.
"""
import json
import os

import numpy as np
import pytest

import oracle
import synth_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "quantize_cases.json")


def _codes(packed):
    """Nibbles of each row in k order, decoded with plain numpy bit operations."""
    lo = (packed & 0x0F).astype(np.int64)
    hi = (packed >> 4).astype(np.int64)
    out = np.empty((packed.shape[0], packed.shape[1] * 2), dtype=np.int64)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out


def _scales_f64(scales):
    return scales.view(np.float16).astype(np.float64)


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_golden(case):
    w = np.array([int(v, 16) for v in case["w"]], dtype=np.uint32).view(np.float32).reshape(1, 32)
    packed, scales, flags = oracle.quantize(w)
    assert packed.tobytes().hex() == case["bytes"]
    assert "%04x" % int(scales[0, 0]) == case["scale"]
    assert flags == case["flags"]


def test_exact_grid_reconstruction():
    rng = np.random.default_rng(11)
    N, K = 64, 256
    G = K // 32
    q = rng.integers(-7, 8, size=(N, K))
    # force max |q| = 7 in every group so amax/7 is exactly the chosen scale
    q.reshape(N, G, 32)[:, :, 0] = rng.choice([-7, 7], size=(N, G))
    # scales: binary16 normals whose 7x multiple is exact in f32
    sbits = rng.integers(0x0400, 0x7000, size=(N, G)).astype(np.uint16)
    s = sbits.view(np.float16).astype(np.float32)
    w = (q.reshape(N, G, 32) * s[:, :, None]).astype(np.float32).reshape(N, K)
    packed, scales, flags = oracle.quantize(w)
    assert flags == 0
    assert np.array_equal(scales, sbits)
    assert np.array_equal(_codes(packed) - 8, q)
    assert np.array_equal(oracle.dequantize(packed, scales), w.astype(np.float64))


def _quantize_random(kind, N, K, seed=0):
    W = synth_inputs.weights(kind, N, K, seed)
    return (W,) + oracle.quantize(W)


@pytest.mark.parametrize("kind", ["normal", "outliers", "student_t", "lm_head"])
def test_round_trip_bound_and_structure(kind):
    W, packed, scales, flags = _quantize_random(kind, 1024, 2560)
    assert flags == 0
    N, K = W.shape
    s = _scales_f64(scales)
    codes = _codes(packed)
    deq = oracle.dequantize(packed, scales)
    # |w - w'| <= s/2 wherever the scale is a binary16 normal
    err = np.abs(W.astype(np.float64) - deq).reshape(N, K // 32, 32)
    normal = s >= 2.0 ** -14
    assert np.all(err[normal] <= (s[normal] / 2)[..., None] * (1 + 2.0 ** -20))
    # every normal-scale group reaches +-7 and never uses code -8
    c = codes.reshape(N, K // 32, 32)
    assert np.all(np.any((c == 1) | (c == 15), axis=2)[normal])
    assert not np.any((c == 0)[normal])
    # scale = binary16(f32(amax) / 7), through numpy's own casts
    amax = np.abs(W).reshape(N, K // 32, 32).max(axis=2)
    want = (amax / np.float32(7.0)).astype(np.float32).astype(np.float16).view(np.uint16)
    assert np.array_equal(scales, want)
    # zero groups: scale 0 and all bytes 0x88
    zero = scales == 0
    if kind == "lm_head":
        assert zero.sum() == (N + 1023) // 1024
    assert np.all(packed.reshape(N, K // 32, 16)[zero] == 0x88)


def test_nearest_integer_characterisation():
    W, packed, scales, _ = _quantize_random("outliers", 512, 1024, seed=3)
    N, K = W.shape
    sf = _scales_f64(scales)
    codes = (_codes(packed) - 8).reshape(N, K // 32, 32)
    t64 = W.astype(np.float64).reshape(N, K // 32, 32) / np.where(sf == 0, 1.0, sf)[..., None]
    cand = np.arange(-8, 8)
    d = np.abs(t64[..., None] - cand)
    best = cand[np.argmin(d, axis=-1)]            # first (lower) candidate on exact ties
    t32 = t64.astype(np.float32).astype(np.float64)
    tie = (t32 - np.floor(t32)) == 0.5
    live = (sf != 0)[..., None] & ~tie
    assert np.array_equal(codes[live], best[live])
    # where the f32 quotient is an exact half, the even neighbour is taken
    tv = t32[tie & (sf != 0)[..., None]]
    if tv.size:
        even = np.where(np.floor(tv) % 2 == 0, np.floor(tv), np.ceil(tv))
        assert np.array_equal(codes[tie & (sf != 0)[..., None]], np.clip(even, -8, 7))


def test_subnormal_scales_clamped_bound():
    rng = np.random.default_rng(5)
    N, K = 256, 64
    # amax spread over the binary16 subnormal-scale range (7 * 2^-25 .. 7 * 2^-14)
    amax = 7.0 * 2.0 ** rng.uniform(-25.5, -14, size=(N, K // 32))
    w = (rng.uniform(-1, 1, size=(N, K // 32, 32)) * amax[..., None]).astype(np.float32)
    w[:, :, 0] = amax.astype(np.float32)
    w = w.reshape(N, K)
    packed, scales, flags = oracle.quantize(w)
    assert flags == 0
    s = _scales_f64(scales)
    deq = oracle.dequantize(packed, scales).reshape(N, K // 32, 32)
    codes = (_codes(packed) - 8).reshape(N, K // 32, 32)
    assert np.all(np.abs(codes) <= 8) and codes.max() <= 7
    t = w.astype(np.float64).reshape(N, K // 32, 32) / np.where(s == 0, 1, s)[..., None]
    inside = (t >= -8.5) & (t <= 7.5) & (s != 0)[..., None]
    err = np.abs(w.reshape(N, K // 32, 32) - deq)
    assert np.all(err[inside] <= (np.broadcast_to(s[..., None], err.shape)[inside] / 2))
    # outside the representable range the code is the clamp end
    assert np.all(codes[(t > 7.5) & (s != 0)[..., None]] == 7)
    assert np.all(codes[(t < -8.5) & (s != 0)[..., None]] == -8)
    assert np.all(deq[s == 0] == 0)


def test_rejects_bad_k():
    with pytest.raises(ValueError):
        oracle.quantize(np.zeros((2, 48), np.float32))


def test_flags_accumulate_over_groups():
    w = np.zeros((3, 64), np.float32)
    w[0, 5] = np.nan
    w[2, 40] = 65520.0 * 7
    w[1, :] = 1.0
    packed, scales, flags = oracle.quantize(w)
    assert flags == oracle.FLAG_NONFINITE | oracle.FLAG_SCALE_OVERFLOW
    assert scales[0, 0] == 0 and scales[2, 1] == 0 and scales[1, 0] == 0x3092


# ---- property test over arbitrary finite float32 groups (hypothesis) ----------------------
from hypothesis import given, settings, strategies as st  # noqa: E402
from hypothesis.extra.numpy import arrays  # noqa: E402


def _check_groups(w):
    """Every group of w against definitions that do not use the oracle's float32 quotient:
    the scale is numpy's binary16 cast of float32(amax) / 7 (a zero group, flagged, when
    that overflows; a zero group when it is zero), and each code is the binary64 nearest
    integer to w / s clamped to [-8, 7], except within 2^-19 of a half (where the float32
    quotient's rounding decides) and within 2^-19 of a clamp end."""
    packed, scales, flags = oracle.quantize(w)
    G = w.shape[1] // 32
    g32 = w.reshape(w.shape[0], G, 32)
    amax = np.max(np.abs(g32), axis=2)                       # float32
    with np.errstate(over="ignore"):
        s16 = (amax / np.float32(7.0)).astype(np.float16)    # numpy's round-to-nearest-even cast
    overflow = np.isinf(s16)
    assert flags == (oracle.FLAG_SCALE_OVERFLOW if overflow.any() else 0)
    codes = (_codes(packed) - 8).reshape(g32.shape)
    zero = overflow | (s16 == 0)
    assert np.all(scales[zero] == 0) and np.all(codes[zero] == 0)
    live = ~zero
    assert np.array_equal(scales[live], s16[live].view(np.uint16))
    sf = np.where(live, s16.astype(np.float64), 1.0)
    t = g32.astype(np.float64) / sf[..., None]
    near = np.clip(np.rint(t), -8, 7)
    frac = np.abs(t - np.floor(t) - 0.5)
    decided = live[..., None] & (frac > 2.0 ** -19) & (np.abs(t - 7.5) > 2.0 ** -19) & (np.abs(t + 8.5) > 2.0 ** -19)
    assert np.array_equal(codes[decided], near[decided])
    # codes that the binary64 rule leaves open are one of the neighbours of the clamped quotient
    open_ = live[..., None] & ~decided
    assert np.all(np.abs(codes[open_] - np.clip(t[open_], -8, 7)) <= 0.5 + 2.0 ** -18)


@st.composite
def _wide_groups(draw):
    """4 x 64 float32 weights, each group m_i 2^(e + d_i): mantissas uniform in [-1, 1] from a
    drawn seed, a drawn group exponent e in [-27, 20] and offsets d_i in [-spread, 0] (spread
    drawn up to 40), so that groups reach zero, subnormal and overflowing scales and hold
    values many binades below their maximum."""
    rng = np.random.default_rng(draw(st.integers(0, 2 ** 32 - 1)))
    e = np.array(draw(st.lists(st.integers(-27, 20), min_size=8, max_size=8)), dtype=np.float64)
    spread = draw(st.integers(0, 40))
    m = rng.uniform(-1.0, 1.0, (4, 64))
    d = rng.integers(-spread, 1, (4, 64))
    return (m * np.exp2(np.repeat(e.reshape(4, 2), 32, axis=1) + d)).astype(np.float32)


@settings(max_examples=300, deadline=None)
@given(_wide_groups())
def test_property_wide_range_groups(w):
    _check_groups(w)


@settings(max_examples=200, deadline=None)
@given(arrays(np.float32, (2, 64), elements=st.floats(width=32, allow_nan=False, allow_infinity=False)))
def test_property_any_finite_float32(w):
    _check_groups(w)
