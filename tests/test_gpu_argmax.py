"""GPU parity of q4_gemv_argmax (greedy LM-head step in one launch) against the oracle.

The GPU's logits are f32 sums, so where two logits are closer than the f32 error an
argmax may legitimately pick either: the checks are (a) the chosen row's exact logit is
within that error of the true maximum, (b) the returned value is the chosen row's logit
to the same error, (c) planted clear winners and exact ties give the exact index."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs
from tests._parity import to_dev_x

pytestmark = pytest.mark.gpu


def _dev(packed, scales):
    return torch.from_numpy(packed).cuda(), torch.from_numpy(scales.view(np.int16)).cuda()


def _check(x, packed, scales, x_dtype, logits=True):
    import bit_weight_only_quantize_b200 as q4
    ws = torch.zeros(q4._lib.load().q4_gemv_argmax_workspace_size(), dtype=torch.uint8, device="cuda")
    idx, val, y = q4.gemv_argmax(to_dev_x(x), *_dev(packed, scales), logits=logits, workspace=ws)
    torch.cuda.synchronize()
    assert torch.count_nonzero(ws).item() == 0                 # the workspace is left zero
    ref = oracle.matmul(x, packed, scales, threads=8)
    idx, val = idx.cpu().numpy(), val.cpu().numpy().astype(np.float64)
    tol = (2e-3 if x_dtype == "f32" else 1e-2) * np.abs(ref).max()
    rows = np.arange(ref.shape[0])
    assert np.all(ref[rows, idx] >= ref.max(axis=1) - tol)
    assert np.all(np.abs(val - ref[rows, idx]) <= tol)
    if y is not None:
        y = y.cpu().numpy()
        assert np.array_equal(y[rows, idx], val.astype(np.float32))    # value is the chosen logit
        assert np.all(y.max(axis=1) == val.astype(np.float32))         # and the largest one
    return idx, ref


@pytest.mark.parametrize("M,N,K,x_dtype", [(1, 50000, 2560, "bf16"), (1, 30000, 1024, "f32"),
                                           (4, 10000, 512, "bf16"), (16, 3001, 256, "bf16"), (2, 1, 256, "bf16")])
def test_matches_oracle(M, N, K, x_dtype):
    packed, scales, _ = oracle.quantize(synth_inputs.weights("outliers", N, K, seed=N + M))
    x = synth_inputs.activations(M, K, x_dtype, seed=M)
    _check(x, packed, scales, x_dtype, logits=(M % 2 == 0))


def test_lm_head_planted_winners():
    w = synth_inputs.LM_HEAD
    W = synth_inputs.weights(w.weights, w.N, w.K, seed=0)
    x = synth_inputs.activations(2, w.K, "bf16", seed=1)
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    winners = [123457, 248319]
    for m, r in enumerate(winners):
        W[r] = np.sign(xf[m]) * 0.1                    # a logit far above every other
    packed, scales, _ = oracle.quantize(W)
    idx, _ = _check(x, packed, scales, "bf16", logits=False)
    assert idx.tolist() == winners


def test_ties_take_the_lowest_row():
    N, K = 4096, 512
    W = synth_inputs.weights("normal", N, K, seed=4) * 0.1
    x = synth_inputs.activations(1, K, "bf16", seed=5)
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    for r in (3 + 16 * 40, 3 + 16 * 7, 3 + 16 * 200):  # the same lane position in three row blocks
        W[r] = np.sign(xf[0]) * 0.05
    packed, scales, _ = oracle.quantize(W)
    idx, _ = _check(x, packed, scales, "bf16")
    assert idx[0] == 3 + 16 * 7
