"""Pins for the oracle's fused gate+up, y = silu(x . dequant(Wg)^T) * (x . dequant(Wu)^T).

Checked against a composition of independent pieces (a binary64 torch matmul of
weights decoded by plain numpy bit operations, and scipy's logistic function
``expit``), and against facts that fix the activation and the roles of the two
matrices: a zero gate gives exactly zero, a large positive gate passes g * u
through unchanged, a large negative gate gives almost zero, and the result is
linear in the up projection but not in the gate.
"""
import numpy as np
import pytest
import torch
from scipy.special import expit

import oracle
import synth_inputs


def _numpy_decode(packed, scales):
    N, K = packed.shape[0], packed.shape[1] * 2
    codes = np.empty((N, K), dtype=np.float64)
    codes[:, 0::2] = (packed & 0x0F).astype(np.float64) - 8
    codes[:, 1::2] = (packed >> 4).astype(np.float64) - 8
    return codes * np.repeat(scales.view(np.float16).astype(np.float64), 32, axis=1)


def _q(kind, N, K, seed):
    packed, scales, _ = oracle.quantize(synth_inputs.weights(kind, N, K, seed=seed))
    return packed, scales


def _x64(x):
    return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64) if x.dtype == np.uint16 else \
        x.astype(np.float64)


@pytest.mark.parametrize("M,N,K,x_dtype", [(1, 64, 256, "f32"), (3, 40, 2560, "bf16"), (16, 17, 96, "bf16")])
def test_matches_independent_composition(M, N, K, x_dtype):
    gate, up = _q("outliers", N, K, 1), _q("normal", N, K, 2)
    x = synth_inputs.activations(M, K, x_dtype, seed=3)
    xt = torch.from_numpy(_x64(x))
    g = (xt @ torch.from_numpy(_numpy_decode(*gate)).T).numpy()
    u = (xt @ torch.from_numpy(_numpy_decode(*up)).T).numpy()
    want = g * expit(g) * u
    got = oracle.gate_up(x, gate, up, threads=4)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def _const_rows(code, scale_bits, N, K):
    """Every weight (code - 8) * scale: one byte value and one scale for the whole matrix."""
    packed = np.full((N, K // 2), code | (code << 4), dtype=np.uint8)
    scales = np.full((N, K // 32), scale_bits, dtype=np.uint16)
    return packed, scales


def test_zero_gate_gives_exact_zero():
    K, N = 64, 8
    x = synth_inputs.activations(2, K, "f32", seed=5)
    y = oracle.gate_up(x, _const_rows(8, 0x3C00, N, K), _q("normal", N, K, 6))   # gate codes 8: w = 0
    assert np.all(y == 0.0)


def test_large_gate_passes_product_and_negative_gate_closes():
    # x = 1 everywhere, gate weights (15 - 8) * 1.0 -> g = 7 K; up weights (9 - 8) * 0.5 -> u = K / 2
    K, N = 64, 4
    x = np.ones((1, K), dtype=np.float32)
    up = _const_rows(9, 0x3800, N, K)
    y = oracle.gate_up(x, _const_rows(15, 0x3C00, N, K), up)
    g, u = 7.0 * K, 0.5 * K
    assert np.all(y == g * u)                              # sigmoid(448) is 1 in binary64
    y_neg = oracle.gate_up(x, _const_rows(1, 0x3C00, N, K), up)          # g = -7 K
    assert np.all(y_neg < 0) and np.all(np.abs(y_neg) < 1e-150)


def test_linear_in_up_not_in_gate():
    K, N = 256, 12
    x = synth_inputs.activations(1, K, "f32", seed=7)
    gate, up = _q("normal", N, K, 8), _q("normal", N, K, 9)
    y = oracle.gate_up(x, gate, up)
    up2 = (up[0], (up[1].view(np.float16) * np.float16(2)).view(np.uint16))   # scales x 2 (exact)
    assert np.array_equal(oracle.gate_up(x, gate, up2), 2.0 * y)
    gate2 = (gate[0], (gate[1].view(np.float16) * np.float16(2)).view(np.uint16))
    assert not np.allclose(oracle.gate_up(x, gate2, up), 2.0 * y, rtol=1e-3)


def test_rows_subset_and_shape_checks():
    K, N = 96, 20
    x = synth_inputs.activations(2, K, "bf16", seed=11)
    gate, up = _q("normal", N, K, 12), _q("normal", N, K, 13)
    full = oracle.gate_up(x, gate, up)
    rows = np.array([19, 0, 7], dtype=np.int64)
    assert np.array_equal(oracle.gate_up(x, gate, up, rows=rows), full[:, rows])
    with pytest.raises(ValueError):
        oracle.gate_up(x, gate, _q("normal", N + 1, K, 14))
