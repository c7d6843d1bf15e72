"""CPU checks of the error bounds the GPU parity tests hold the kernels to (tests/_parity.py).

A bound that is too tight fails good kernels; one that is too loose hides bad ones.  These
tests pin the bound helpers to facts that do not depend on them: the defining inequality of
the power-of-two shift, the exact rounding error of x on that grid (computed in binary64
from its definition), and the classical bound on a sequential float32 sum, checked against
numpy's own float32 additions (round to nearest) and against sums rounded toward zero (the
model the tests take for sums inside a tensor-core instruction)."""
import numpy as np
import pytest

import oracle
import synth_inputs
from tests._parity import (U_CUDA_CORE, U_TENSOR_F32, digit_path_bound, digit_shift, f32_sum_bound,
                           gamma, mma_path_bound, x_f64)


@pytest.mark.parametrize("mx", [1.0, 2.0, 0.5, 3.0, 2.0 ** 29, 2.0 ** -60, 1.0 - 2.0 ** -24, 1.5 * 2.0 ** -20,
                                np.float32(3.3e-5), 7.0e4])
def test_digit_shift_is_the_largest_shift_below_2_30(mx):
    """F is the largest integer with max|x| * 2^F < 2^30 (capped at 100)."""
    x = np.array([0.25 * mx, -mx, 0.0], dtype=np.float64)
    F = digit_shift(x)
    assert mx * 2.0 ** F < 2.0 ** 30
    assert F == 100 or mx * 2.0 ** (F + 1) >= 2.0 ** 30


def test_digit_shift_degenerate_boxes():
    assert digit_shift(np.zeros(256)) == 100
    assert digit_shift(np.full(256, 2.0 ** -130)) == 100   # below the smallest normal f32
    assert digit_shift(np.array([])) == 100


def test_digit_bound_covers_the_rounding_of_x_to_the_box_grid():
    """The first term of the M = 1 bound, sum_k |w'_k| 2^(-F-1), must cover the exact error
    of replacing x by rint(x 2^F) 2^-F box by box, with no float32 sum involved."""
    K, N = 1024, 40
    W = synth_inputs.weights("outliers", N, K, seed=11)
    packed, scales, _ = oracle.quantize(W)
    deq = oracle.dequantize(packed, scales)

    def grid_error(x):
        xs = x_f64(x)[0]
        xr = np.empty_like(xs)
        for b in range(0, K, 256):
            F = digit_shift(xs[b:b + 256])
            xr[b:b + 256] = np.rint(xs[b:b + 256] * 2.0 ** F) * 2.0 ** -F
        return np.abs(deq @ (xs - xr))

    # f32 x: 24 significant bits do not fit the grid below max|x| / 2^6
    x = synth_inputs.activations(1, K, "f32", seed=12)
    err = grid_error(x)
    zero_sum_bound = digit_path_bound(x, deq, 0)[0]         # n = 0: only the rounding of x
    assert np.all(err <= zero_sum_bound)
    assert np.all(err > 0.0)
    # and the bound is not vacuous: within a small factor of what rounding can reach
    assert np.max(err / zero_sum_bound) > 1e-3
    # bf16 x: 8 significant bits land on the grid unless a box spans more than 22 binades
    xb = synth_inputs.activations(1, K, "bf16", seed=12)
    assert np.all(grid_error(xb) == 0.0)


def _sequential_f32(terms: np.ndarray, toward_zero: bool) -> np.ndarray:
    """Sum terms[:, k] over k in float32, one rounding per addition."""
    acc = np.zeros(terms.shape[0], dtype=np.float32)
    for k in range(terms.shape[1]):
        exact = acc.astype(np.float64) + terms[:, k].astype(np.float64)   # exact for these terms
        r = exact.astype(np.float32)
        if toward_zero:
            over = np.abs(r.astype(np.float64)) > np.abs(exact)
            r[over] = np.nextafter(r[over], np.float32(0.0))
        acc = r
    return acc


@pytest.mark.parametrize("toward_zero", [False, True])
def test_f32_sum_bounds_cover_sequential_sums(toward_zero):
    """Exact products of bf16 x and (code - 8) * scale summed over K in one float32 chain:
    the error against the binary64 oracle stays within gamma_K(u) sum |x w'|, u = 2^-24 for
    round to nearest, 2^-23 for round toward zero."""
    K, N = 512, 64
    W = np.abs(synth_inputs.weights("normal", N, K, seed=21))  # same-sign terms: the errors add up
    packed, scales, _ = oracle.quantize(W)
    deq = oracle.dequantize(packed, scales)
    x = synth_inputs.activations(1, K, "bf16", seed=22)
    x = x & np.uint16(0x7FFF)                                  # |x|, still bf16 bits
    terms = (x_f64(x)[0][None, :] * deq).astype(np.float32)
    assert np.array_equal(terms.astype(np.float64), x_f64(x)[0][None, :] * deq)   # products exact
    ref = oracle.matmul(x, packed, scales, threads=1)[0]
    y = _sequential_f32(terms, toward_zero)
    err = np.abs(y.astype(np.float64) - ref)
    bound = (mma_path_bound if toward_zero else f32_sum_bound)(x, deq, K)[0]
    assert np.all(err <= bound)
    # truncation loses on every addition, so its error is a sizeable part of the bound
    if toward_zero:
        assert np.max(err / bound) > 0.05


@pytest.mark.parametrize("toward_zero", [False, True])
def test_worst_case_chain_reaches_the_bound(toward_zero):
    """1 followed by n terms just below one ulp of 1 (round toward zero) or just below half an
    ulp (round to nearest): every addition drops its whole term, so the error approaches
    gamma_n(u) sum |terms| with the model's u, and the other model's u would be too small
    by a factor of two for truncation."""
    n = 1000
    t = np.float32((0.99 if toward_zero else 0.495) * 2.0 ** -23)
    terms = np.concatenate([[np.float32(1.0)], np.full(n, t, dtype=np.float32)])[None, :]
    y = _sequential_f32(terms, toward_zero)[0]
    assert y == np.float32(1.0)                               # every term was dropped
    exact = 1.0 + n * float(t)
    err = exact - float(y)
    u = U_TENSOR_F32 if toward_zero else U_CUDA_CORE
    bound = gamma(n, u) * exact
    assert err <= bound
    assert err >= 0.95 * bound                                # the bound is tight here
    if toward_zero:
        assert err > gamma(n, U_CUDA_CORE) * exact            # 2^-24 would not cover truncation


def test_unit_roundoffs_and_gamma():
    assert U_CUDA_CORE == np.finfo(np.float32).eps / 2
    assert U_TENSOR_F32 == np.finfo(np.float32).eps
    assert gamma(0, U_CUDA_CORE) == 0.0
    assert gamma(3, 0.5 ** 10) == 3 * 0.5 ** 10 / (1 - 3 * 0.5 ** 10)
