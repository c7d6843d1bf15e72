"""Pins for the oracle's INT8 weight format (the INT8 half of a mixed INT8/INT4 model,
QKV-Core thread, section "自适应混合量化"; the encoding is this library's reading, written
out in q4_oracle.c): s = binary16(amax / 127), q = clamp(rint(w / s), -128, 127), w' = q * s.

Checked against facts that do not go through the oracle's own code: the round-trip bound
|w - w'| <= s/2 against the stored scale, exact reconstruction of weights already on the
grid, zero groups, the clamp reached only through a binary16 scale rounded down, flags for
non-finite input and scale overflow, and products against numpy's binary16 decoding with a
torch binary64 matmul and a hand-summed brute force; and (hypothesis) the scale and
nearest-integer rules on arbitrary finite float32 groups spanning every binade."""
import numpy as np
import pytest
import torch
from fractions import Fraction

import oracle
import synth_inputs


def _np_decode(codes, scales):
    s = scales.view(np.float16).astype(np.float64)             # numpy's binary16, not the oracle's
    return codes.astype(np.float64) * np.repeat(s, 32, axis=1)


@pytest.mark.parametrize("kind", ["normal", "outliers", "student_t"])
def test_round_trip_bound_against_stored_scale(kind):
    W = synth_inputs.weights(kind, 64, 512, seed=3)
    codes, scales, flags = oracle.quantize8(W)
    assert flags == 0
    s = np.repeat(scales.view(np.float16).astype(np.float64), 32, axis=1)
    deq = _np_decode(codes, scales)
    inside = (codes > -128) & (codes < 127)                     # not clamped
    assert np.all(np.abs(W.astype(np.float64) - deq)[inside] <= s[inside] / 2)
    assert np.array_equal(deq, oracle.dequantize8(codes, scales))
    # the largest magnitude of every group maps to code +-127 (the divisor is 127)
    amax_code = np.abs(codes.reshape(64, -1, 32).astype(np.int32)).max(axis=2)
    assert np.all(amax_code == 127)


def test_weights_on_the_grid_come_back_exactly():
    rng = np.random.default_rng(5)
    c = rng.integers(-127, 128, size=(8, 256))
    c[:, ::32] = 127                                            # amax code 127 in every group
    W = (c * 2.0 ** -7).astype(np.float32)                      # s = 2^-7 exactly
    codes, scales, flags = oracle.quantize8(W)
    assert flags == 0 and np.all(scales == np.float16(2.0 ** -7).view(np.uint16))
    assert np.array_equal(codes, c.astype(np.int8))
    assert np.array_equal(_np_decode(codes, scales), W.astype(np.float64))


def test_zero_groups_and_flags():
    W = synth_inputs.weights("normal", 4, 128, seed=6)
    W[0, 32:64] = 0.0                                           # zero group
    W[1, 0] = np.nan                                            # non-finite
    W[2, 64:96] = 1.0e7                                         # 1e7 / 127 overflows binary16
    codes, scales, flags = oracle.quantize8(W)
    assert flags == 3
    for n, g in ((0, 1), (1, 0), (2, 2)):
        assert scales[n, g] == 0 and np.all(codes[n, 32 * g:32 * g + 32] == 0)
    x = synth_inputs.activations(1, 128, "f32", seed=7)
    W2 = W.copy()
    W2[1, 0:32] = 0.0
    W2[2, 64:96] = 0.0
    ref = oracle.matmul8(x, codes, scales)
    assert np.allclose(ref, oracle.matmul8(x, *oracle.quantize8(W2)[:2]), rtol=0, atol=0)


def test_clamp_reached_only_through_a_rounded_down_subnormal_scale():
    # amax = 127 * 1.4 * 2^-24: s32 = 1.4 * 2^-24 rounds to the subnormal 2^-24, so
    # -amax / s = -177.8 clamps to -128 and +amax to +127
    a = np.float32(127 * 1.4 * 2.0 ** -24)
    W = np.zeros((1, 32), dtype=np.float32)
    W[0, 0], W[0, 1] = -a, a
    codes, scales, _ = oracle.quantize8(W)
    assert scales[0, 0] == 1                                    # binary16 bits of 2^-24
    assert codes[0, 0] == -128 and codes[0, 1] == 127


def test_products_against_independent_decoding():
    M, N, K = 3, 40, 2560
    codes, scales, _ = oracle.quantize8(synth_inputs.weights("outliers", N, K, seed=8))
    for dt in ("f32", "bf16"):
        x = synth_inputs.activations(M, K, dt, seed=9)
        xd = (x.astype(np.uint32) << 16).view(np.float32) if dt == "bf16" else x
        want = (torch.from_numpy(xd.astype(np.float64)) @ torch.from_numpy(_np_decode(codes, scales)).T).numpy()
        got = oracle.matmul8(x, codes, scales, threads=4)
        assert np.allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_brute_force_dot_products_k32_k64():
    rng = np.random.default_rng(10)
    for K in (32, 64):
        c = rng.integers(-127, 128, size=(2, K))
        c[:, ::32] = 127
        W = (c * 2.0 ** -6).astype(np.float32)
        x = rng.integers(-8, 9, size=(1, K)).astype(np.float32) / 4
        codes, scales, _ = oracle.quantize8(W)
        y = oracle.matmul8(x, codes, scales)
        for n in range(2):
            exact = sum(Fraction(float(x[0, k])) * Fraction(int(c[n, k])) * Fraction(1, 64) for k in range(K))
            assert y[0, n] == float(exact)


# ---- property test over arbitrary finite float32 groups (hypothesis) ----------------------
from hypothesis import given, settings, strategies as st  # noqa: E402
from hypothesis.extra.numpy import arrays  # noqa: E402

from tests.test_oracle_quantize import _wide_groups  # noqa: E402


def _check_groups8(w):
    """Every group against definitions that do not use the oracle's float32 quotient: the
    scale is numpy's binary16 cast of float32(amax) / 127 (zero group when it is zero or,
    flagged, when it overflows) and each code is the binary64 nearest integer to w / s
    clamped to [-128, 127], except within 2^-15 of a half or of a clamp end (float32
    quotients near 128 carry ulps of 2^-16)."""
    codes, scales, flags = oracle.quantize8(w)
    G = w.shape[1] // 32
    g32 = w.reshape(w.shape[0], G, 32)
    amax = np.max(np.abs(g32), axis=2)
    with np.errstate(over="ignore"):
        s16 = (amax / np.float32(127.0)).astype(np.float16)
    overflow = np.isinf(s16)
    assert flags == (oracle.FLAG_SCALE_OVERFLOW if overflow.any() else 0)
    c = codes.astype(np.int64).reshape(g32.shape)
    zero = overflow | (s16 == 0)
    assert np.all(scales[zero] == 0) and np.all(c[zero] == 0)
    live = ~zero
    assert np.array_equal(scales[live], s16[live].view(np.uint16))
    t = g32.astype(np.float64) / np.where(live, s16.astype(np.float64), 1.0)[..., None]
    near = np.clip(np.rint(t), -128, 127)
    eps = 2.0 ** -15
    decided = (live[..., None] & (np.abs(t - np.floor(t) - 0.5) > eps) & (np.abs(t - 127.5) > eps) &
               (np.abs(t + 128.5) > eps))
    assert np.array_equal(c[decided], near[decided])
    open_ = live[..., None] & ~decided
    assert np.all(np.abs(c[open_] - np.clip(t[open_], -128, 127)) <= 0.5 + 2 * eps)


@settings(max_examples=300, deadline=None)
@given(_wide_groups())
def test_property_wide_range_groups(w):
    _check_groups8(w)


@settings(max_examples=200, deadline=None)
@given(arrays(np.float32, (2, 64), elements=st.floats(width=32, allow_nan=False, allow_infinity=False)))
def test_property_any_finite_float32(w):
    _check_groups8(w)
