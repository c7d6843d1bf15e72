"""GPU parity of q4_quantize against the oracle: packed bytes, scales and flags bit-exact."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth_inputs
from tests._parity import to_dev_f32, to_np_u8, to_np_u16

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "quantize_cases.json")


def gpu_quantize(W: np.ndarray):
    import bit_weight_only_quantize_b200 as q4
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    packed, scales = q4.quantize(to_dev_f32(W), flags)
    torch.cuda.synchronize()
    return to_np_u8(packed), to_np_u16(scales), int(flags.item())


def assert_same(W):
    gp, gs, gf = gpu_quantize(W)
    op, os_, of = oracle.quantize(W)
    assert np.array_equal(gp, op)
    assert np.array_equal(gs, os_)
    assert gf == of


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_golden_cases(case):
    w = np.array([int(v, 16) for v in case["w"]], dtype=np.uint32).view(np.float32).reshape(1, 32)
    gp, gs, gf = gpu_quantize(w)
    assert gp.tobytes().hex() == case["bytes"]
    assert "%04x" % int(gs[0, 0]) == case["scale"]
    assert gf == case["flags"]


@pytest.mark.parametrize("N,K", [(1, 32), (3, 96), (37, 160), (129, 2592), (1000, 1024), (7, 8192)])
def test_ragged_shapes(N, K):
    assert_same(synth_inputs.weights("outliers", N, K, seed=N + K))


@pytest.mark.parametrize("w", [w for w in synth_inputs.ALL if w.op == "gemv" and w.N <= 4096]
                         + [synth_inputs.PREFILL[0]], ids=lambda w: w.name)
def test_config_shapes(w):
    assert_same(synth_inputs.weights(w.weights, w.N, w.K, seed=0))


def test_lm_head_full():
    w = synth_inputs.LM_HEAD
    assert_same(synth_inputs.weights(w.weights, w.N, w.K, seed=0))


def test_random_bit_patterns_flags():
    rng = np.random.default_rng(9)
    W = rng.integers(0, 2 ** 32, size=(64, 256), dtype=np.uint64).astype(np.uint32).view(np.float32)
    assert_same(W)
    _, _, f = oracle.quantize(W)
    assert f == oracle.FLAG_NONFINITE | oracle.FLAG_SCALE_OVERFLOW


def test_subnormal_scale_range():
    rng = np.random.default_rng(10)
    N, K = 512, 256
    amax = 7.0 * 2.0 ** rng.uniform(-26, -13, size=(N, K // 32))
    W = (rng.uniform(-1, 1, size=(N, K // 32, 32)) * amax[..., None]).astype(np.float32)
    W[:, :, 3] = -amax.astype(np.float32)
    assert_same(W.reshape(N, K))


def test_ties_and_negative_zero():
    # quotients landing exactly on k + 1/2 with power-of-two scales
    rng = np.random.default_rng(12)
    N, K = 64, 128
    s = 2.0 ** rng.integers(-10, 4, size=(N, K // 32, 1))
    t = rng.integers(-15, 15, size=(N, K // 32, 32)) / 2.0
    t[:, :, 0] = 7.0
    W = (t * s).astype(np.float32).reshape(N, K)
    W[0, 1] = -0.0
    assert_same(W)


def test_flags_are_ored_not_cleared():
    import bit_weight_only_quantize_b200 as q4
    flags = torch.full((1,), 4, dtype=torch.int32, device="cuda")
    W = np.zeros((2, 64), np.float32)
    W[1, 0] = np.inf
    q4.quantize(to_dev_f32(W), flags)
    torch.cuda.synchronize()
    assert int(flags.item()) == 4 | oracle.FLAG_NONFINITE


def test_empty():
    import bit_weight_only_quantize_b200 as q4
    packed, scales = q4.quantize(torch.zeros((0, 64), device="cuda"))
    assert packed.shape == (0, 32) and scales.shape == (0, 2)
