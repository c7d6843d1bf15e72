"""Pins for the oracle products y = x . dequant(W)^T.

Checked against hand-computed dot products (tests/golden/product_cases.json),
a binary64 torch matmul of weights decoded by plain numpy bit operations
(a library routine on an independent decode), and structural facts (zero rows,
row subsets, bf16 widening).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "product_cases.json")


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_golden(case):
    K, N, M = case["K"], case["N"], case["M"]
    packed = np.array([list(bytes.fromhex(r)) for r in case["packed"]], dtype=np.uint8).reshape(N, K // 2)
    scales = np.array([[int(v, 16) for v in r] for r in case["scales"]], dtype=np.uint16).reshape(N, K // 32)
    x = np.array(case["x"], dtype=np.float32).reshape(M, K)
    y = oracle.matmul(x, packed, scales)
    assert np.array_equal(y, np.array(case["y"], dtype=np.float64))


def _numpy_decode(packed, scales):
    N = packed.shape[0]
    K = packed.shape[1] * 2
    codes = np.empty((N, K), dtype=np.float64)
    codes[:, 0::2] = (packed & 0x0F).astype(np.float64) - 8
    codes[:, 1::2] = (packed >> 4).astype(np.float64) - 8
    s = np.repeat(scales.view(np.float16).astype(np.float64), 32, axis=1)
    return codes * s


@pytest.mark.parametrize("x_dtype,M", [("f32", 1), ("bf16", 1), ("bf16", 5), ("f32", 16)])
def test_matches_torch_f64(x_dtype, M):
    W = synth_inputs.weights("outliers", 300, 1024, seed=1)
    packed, scales, _ = oracle.quantize(W)
    x = synth_inputs.activations(M, 1024, x_dtype, seed=1)
    y = oracle.matmul(x, packed, scales, threads=4)
    if x_dtype == "bf16":
        xt = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).double()
    else:
        xt = torch.from_numpy(x).double()
    wd = torch.from_numpy(_numpy_decode(packed, scales))
    assert np.array_equal(oracle.dequantize(packed, scales), wd.numpy())
    ref = (xt @ wd.T).numpy()
    assert np.max(np.abs(y - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_row_subset_and_zero_rows():
    W = synth_inputs.weights("normal", 257, 512, seed=2)
    W[7] = 0.0
    packed, scales, _ = oracle.quantize(W)
    x = synth_inputs.activations(3, 512, "bf16", seed=2)
    full = oracle.matmul(x, packed, scales, threads=2)
    assert np.all(full[:, 7] == 0.0)
    rows = np.array([256, 0, 7, 100, 100], dtype=np.int64)
    sub = oracle.matmul(x, packed, scales, rows=rows)
    assert np.array_equal(sub, full[:, rows])


def test_thread_count_does_not_change_results():
    W = synth_inputs.weights("student_t", 200, 256, seed=4)
    packed, scales, _ = oracle.quantize(W)
    x = synth_inputs.activations(4, 256, "f32", seed=4)
    assert np.array_equal(oracle.matmul(x, packed, scales, threads=1),
                          oracle.matmul(x, packed, scales, threads=8))


def test_bf16_widening_is_exact():
    bits = np.array([[0x3F80, 0xBF80, 0x4049, 0x0001, 0x7F7F] + [0] * 27], dtype=np.uint16)
    packed = np.full((5, 16), 0x88, dtype=np.uint8)
    scales = np.zeros((5, 1), dtype=np.uint16)
    for j in range(5):            # row j: code +1 at k=j, scale 1.0
        b = list(packed[j])
        b[j // 2] = 0x89 if j % 2 == 0 else 0x98
        packed[j] = b
        scales[j, 0] = 0x3C00
    y = oracle.matmul(bits, packed, scales)
    want = (bits[0, :5].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.array_equal(y[0], want)
