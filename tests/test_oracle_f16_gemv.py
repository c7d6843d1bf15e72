"""Pins for the oracle's F16-weight GEMV y = x . W^T (W binary16): a binary64 torch matmul
of numpy's float16 -> float64 widening (library routines), exact hand cases with
power-of-two weights, and structure (zero rows, f32 vs bf16 x)."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs


def _w16(N, K, seed):
    return synth_inputs.weights("normal", N, K, seed=seed).astype(np.float16).view(np.uint16)


@pytest.mark.parametrize("M,N,K,x_dtype", [(1, 64, 256, "f32"), (3, 50, 2560, "bf16"), (16, 7, 96, "bf16")])
def test_matches_torch_f64(M, N, K, x_dtype):
    w16 = _w16(N, K, 1)
    x = synth_inputs.activations(M, K, x_dtype, seed=2)
    xf = (x.astype(np.uint32) << 16).view(np.float32) if x.dtype == np.uint16 else x
    want = (torch.from_numpy(xf.astype(np.float64)) @ torch.from_numpy(w16.view(np.float16).astype(np.float64)).T)
    got = oracle.f16_matmul(x, w16, threads=4)
    assert np.allclose(got, want.numpy(), rtol=1e-13, atol=1e-13)


def test_exact_small_cases():
    # powers of two and small integers: every product and sum is exact
    K = 8
    w = np.array([[1, 2, 4, 8, -1, -2, -4, -8], [0.5, 0.25, 0, 0, 0, 0, 0, 65504]], dtype=np.float16)
    x = np.array([[1, 1, 1, 1, 1, 1, 1, 1], [3, 0, 0, 0, 0, 0, 0, 2]], dtype=np.float32)
    y = oracle.f16_matmul(x, w.view(np.uint16))
    assert y.tolist() == [[0.0, 65504.75], [3.0 - 16.0, 1.5 + 131008.0]]


def test_zero_rows_and_subnormal_weights():
    K, N = 64, 4
    w = np.zeros((N, K), dtype=np.float16)
    w[2, :] = np.float16(2.0 ** -24)                        # smallest binary16 subnormal
    x = np.ones((1, K), dtype=np.float32)
    y = oracle.f16_matmul(x, w.view(np.uint16))
    assert y[0].tolist() == [0.0, 0.0, K * 2.0 ** -24, 0.0]
