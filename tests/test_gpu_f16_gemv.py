"""GPU parity of q4_f16_gemv (binary16 weights on the tensor cores) against the oracle's
binary64 f16_matmul: the stated tolerance, and a per-element bound from the arithmetic
(exact binary16 products of the scaled x, f32 accumulation that may truncate; for f32 x
the 2^-22 relative error of its two-part split)."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs
from tests._parity import rel_inf, to_dev_x

pytestmark = pytest.mark.gpu

TOL = {"f32": 2e-3, "bf16": 1e-2}


def _w16(N, K, seed, kind="normal"):
    K32 = -(-K // 32) * 32                      # the generator draws whole groups of 32
    W = synth_inputs.weights(kind, N, K32, seed=seed)[:, :K]
    return np.ascontiguousarray(W).astype(np.float16).view(np.uint16)


def _x64(x):
    return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64) if x.dtype == np.uint16 else \
        x.astype(np.float64)


def run(M, N, K, x_dtype, seed, kind="normal", static=False):
    import bit_weight_only_quantize_b200 as q4
    w16 = _w16(N, K, seed, kind)
    x = synth_inputs.activations(M, K, x_dtype, seed=seed + 1)
    wd = torch.from_numpy(w16.view(np.int16)).cuda().view(torch.float16)
    y = q4.f16_gemv(to_dev_x(x), wd, weights_static=static)
    torch.cuda.synchronize()
    y = y.cpu().numpy()
    ref = oracle.f16_matmul(x, w16, threads=8)
    assert rel_inf(y, ref) <= TOL[x_dtype]
    n = K // 16 + 8
    u = 2.0 ** -23
    mag = np.abs(_x64(x)) @ np.abs(w16.view(np.float16).astype(np.float64)).T
    bound = n * u / (1 - n * u) * mag + (2.0 ** -22 * mag if x_dtype == "f32" else 0.0)
    assert np.all(np.abs(y - ref) <= bound + 1e-30)
    return y, ref


@pytest.mark.parametrize("x_dtype", ["f32", "bf16"])
@pytest.mark.parametrize("M,N,K", [(1, 1, 8), (1, 17, 72), (1, 100, 2560), (1, 4096, 2560), (1, 33, 136)])
def test_m1(M, N, K, x_dtype):
    run(M, N, K, x_dtype, seed=N + K)


@pytest.mark.parametrize("M,N,K", [(2, 64, 1024), (5, 250, 2560), (8, 31, 520), (9, 300, 256), (16, 4096, 2560)])
def test_small_batch(M, N, K):
    run(M, N, K, "bf16", seed=M * 10 + N, kind="student_t", static=(M % 2 == 1))


def test_large_and_tiny_activations_keep_precision():
    import bit_weight_only_quantize_b200 as q4
    N, K = 64, 512
    w16 = _w16(N, K, 3)
    for scale in (2.0 ** 40, 2.0 ** -60):           # outside binary16's range without the 2^-e_m scaling
        xf = (synth_inputs.activations(1, K, "f32", seed=4) * np.float32(scale)).astype(np.float32)
        xb = xf.view(np.uint32) >> 16              # truncated to bf16 bits
        xb = xb.astype(np.uint16)
        y = q4.f16_gemv(to_dev_x(xb), torch.from_numpy(w16.view(np.int16)).cuda().view(torch.float16))
        ref = oracle.f16_matmul(xb, w16)
        assert rel_inf(y.cpu().numpy(), ref) <= 1e-5


def test_lm_head_rows_sampled():
    """The LM-head shape in binary16 (1.27 GB of weights), checked on sampled rows."""
    import bit_weight_only_quantize_b200 as q4
    N, K = 248320, 2560
    w16 = _w16(N, K, 7)
    x = synth_inputs.activations(1, K, "bf16", seed=8)
    y = q4.f16_gemv(to_dev_x(x), torch.from_numpy(w16.view(np.int16)).cuda().view(torch.float16)).cpu().numpy()
    rows = np.random.default_rng(0).choice(N, 512, replace=False)
    ref = oracle.f16_matmul(x, w16[rows])
    assert rel_inf(y[:, rows], ref) <= 1e-5
