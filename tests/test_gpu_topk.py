"""GPU parity of q4_gemv_topk (the k largest LM-head logits per x row in one launch)
against the oracle.

The GPU's logits are f32 sums, so rows whose logits lie within the f32 error of the k-th
largest may legitimately enter or leave the list.  The checks are: (a) the lists are a
valid top-k of the kernel's own logits (sorted, ties to the lower row, nothing left out
above the last entry); (b) against the oracle's binary64 logits every listed row is
within tolerance of the true k-th largest, every value is within tolerance of the true
logit of its row, and every row clearly inside the true top-k is listed; (c) planted
winners, exact ties, short lists and row offsets give exact indices."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs
from tests._parity import to_dev_x

pytestmark = pytest.mark.gpu


def _dev(packed, scales):
    return torch.from_numpy(packed).cuda(), torch.from_numpy(scales.view(np.int16)).cuda()


def _valid_topk(y, idx, val, k):
    """idx/val is a top-k of the rows of y (f32): sorted, ties to lower rows, complete."""
    M, N = y.shape
    for m in range(M):
        n = min(k, N)
        assert np.all(idx[m, n:] == -1) and np.all(np.isnan(val[m, n:]))
        i, v = idx[m, :n], val[m, :n]
        assert len(set(i.tolist())) == n and np.all((i >= 0) & (i < N))
        assert np.array_equal(v, y[m, i])                                   # values are the logits
        assert np.all((v[:-1] > v[1:]) | ((v[:-1] == v[1:]) & (i[:-1] < i[1:])))   # order and ties
        rest = np.ones(N, dtype=bool)
        rest[i] = False
        last_v, last_i = v[-1], i[-1]
        r = np.nonzero(rest)[0]
        assert np.all((y[m, r] < last_v) | ((y[m, r] == last_v) & (r > last_i)))   # nothing better left out


def _check(x, packed, scales, x_dtype, k, row_base=0, logits=True):
    import bit_weight_only_quantize_b200 as q4
    M, N = x.shape[0], packed.shape[0]
    dx = to_dev_x(x)
    ws = torch.zeros(q4.gemv_topk_workspace_size(M, N, packed.shape[1] * 2, k, dx.dtype), dtype=torch.uint8,
                     device="cuda")
    idx, val, y = q4.gemv_topk(dx, *_dev(packed, scales), k, row_base=row_base, logits=logits, workspace=ws)
    idx2, val2, _ = q4.gemv_topk(dx, *_dev(packed, scales), k, row_base=row_base, workspace=ws)   # reuse
    torch.cuda.synchronize()
    assert torch.count_nonzero(ws[:16]).item() == 0                     # the counter is left zero
    idx, val = idx.cpu().numpy(), val.cpu().numpy()
    assert np.array_equal(idx, idx2.cpu().numpy()) and np.array_equal(val, val2.cpu().numpy(), equal_nan=True)
    loc = np.where(idx >= 0, idx - row_base, -1)
    if y is not None:
        _valid_topk(y.cpu().numpy(), loc, val, k)
    ref = oracle.matmul(x, packed, scales, threads=8)
    tol = (2e-3 if x_dtype == "f32" else 1e-2) * np.abs(ref).max()
    n = min(k, N)
    for m in range(M):
        order = np.lexsort((np.arange(N), -ref[m]))
        kth = ref[m, order[n - 1]]
        assert np.all(ref[m, loc[m, :n]] >= kth - tol)                    # listed rows are near the top
        assert np.all(np.abs(val[m, :n].astype(np.float64) - ref[m, loc[m, :n]]) <= tol)
        sure = order[:n][ref[m, order[:n]] > kth + 2 * tol]               # clearly inside the top k
        assert set(sure.tolist()) <= set(loc[m, :n].tolist())
    return idx, val


@pytest.mark.parametrize("M,N,K,x_dtype,k", [(1, 50000, 2560, "bf16", 20), (1, 30000, 1024, "f32", 20),
                                             (4, 10000, 512, "bf16", 32), (16, 3001, 256, "bf16", 5),
                                             (3, 100, 768, "bf16", 1), (8, 4096, 2560, "bf16", 20)])
def test_matches_oracle(M, N, K, x_dtype, k):
    packed, scales, _ = oracle.quantize(synth_inputs.weights("outliers", N, K, seed=N + M))
    x = synth_inputs.activations(M, K, x_dtype, seed=M)
    _check(x, packed, scales, x_dtype, k, logits=(M != 8))


def test_lm_head_planted_top20():
    w = synth_inputs.LM_HEAD
    W = synth_inputs.weights(w.weights, w.N, w.K, seed=0)
    x = synth_inputs.activations(1, w.K, "bf16", seed=1)
    xf = (x.astype(np.uint32) << 16).view(np.float32)[0]
    planted = [248319, 0, 123457, 77, 200000, 16, 31, 131071, 5000, 99999,
               1, 2, 3, 240000, 17, 18, 33, 65536, 150001, 190000]
    for i, r in enumerate(planted):                       # strictly decreasing, far above the rest
        W[r] = np.sign(xf) * (0.2 - 0.005 * i)
    packed, scales, _ = oracle.quantize(W)
    idx, _ = _check(x, packed, scales, "bf16", 20, logits=False)
    assert idx[0].tolist() == planted


def test_ties_short_lists_and_row_base():
    import bit_weight_only_quantize_b200 as q4
    N, K = 4096, 512
    W = synth_inputs.weights("normal", N, K, seed=4) * 0.1
    x = synth_inputs.activations(1, K, "bf16", seed=5)
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    for r in (3 + 16 * 40, 3 + 16 * 7, 3 + 16 * 200, 3 + 16 * 240):   # equal logits, same lane in four blocks
        W[r] = np.sign(xf[0]) * 0.05
    packed, scales, _ = oracle.quantize(W)
    idx, _ = _check(x, packed, scales, "bf16", 3, row_base=1000)
    assert idx[0].tolist() == [1000 + 3 + 16 * 7, 1000 + 3 + 16 * 40, 1000 + 3 + 16 * 200]
    # fewer rows than k: the tail is -1 / NaN
    p7, s7, _ = oracle.quantize(synth_inputs.weights("normal", 7, 256, seed=6))
    x2 = synth_inputs.activations(2, 256, "bf16", seed=7)
    idx, val = _check(x2, p7, s7, "bf16", 20)
    assert np.all(idx[:, 7:] == -1) and np.all(np.isnan(val[:, 7:]))
    assert sorted(idx[0, :7].tolist()) == list(range(7))
    # N == 0: all padding
    e_idx, e_val, _ = q4.gemv_topk(to_dev_x(x2), torch.zeros((0, 128), dtype=torch.uint8, device="cuda"),
                                   torch.zeros((0, 8), dtype=torch.int16, device="cuda"), 4)
    assert torch.all(e_idx == -1) and torch.all(torch.isnan(e_val))


def test_k1_matches_greedy_argmax():
    import bit_weight_only_quantize_b200 as q4
    packed, scales, _ = oracle.quantize(synth_inputs.weights("outliers", 20000, 1024, seed=8))
    x = to_dev_x(synth_inputs.activations(5, 1024, "bf16", seed=9))
    i1, v1, _ = q4.gemv_topk(x, *_dev(packed, scales), 1)
    ia, va, _ = q4.gemv_argmax(x, *_dev(packed, scales))
    assert torch.equal(i1[:, 0], ia) and torch.equal(v1[:, 0], va)
