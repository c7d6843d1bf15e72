"""GPU parity of q4_topk_merge against the oracle's selection (bit-exact: it is index
work on given f32 values), and of the row-sharded LM head emulated on one GPU: shard
top-k lists from q4_gemv_topk with global rows, merged, checked against the oracle's top
k of the whole head.  (The all-gather of the lists is covered by gloo ranks on CPU.)"""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs
from tests._parity import to_dev_x
from tests.test_gpu_topk import _dev

pytestmark = pytest.mark.gpu


def _lists(S, M, k, seed, pad=0, nan=0):
    """S disjoint row lists per x row, values with deliberate ties, some padding and NaNs."""
    rng = np.random.default_rng(seed)
    vals = rng.integers(-50, 50, size=(S, M, k)).astype(np.float32) * np.float32(0.125)   # many exact ties
    rows = np.stack([np.stack([rng.choice(np.arange(s * 100000, s * 100000 + 5000), size=k, replace=False)
                               for _ in range(M)]) for s in range(S)]).astype(np.int64)
    flat_v, flat_r = vals.reshape(-1), rows.reshape(-1)
    flat_r[rng.choice(flat_r.size, size=pad, replace=False)] = -1
    flat_v[rng.choice(flat_v.size, size=nan, replace=False)] = np.nan
    return vals, rows


@pytest.mark.parametrize("S,M,k,pad,nan", [(8, 1, 20, 0, 0), (2, 16, 32, 5, 0), (5, 3, 7, 20, 3), (1, 4, 1, 0, 1),
                                           (64, 2, 20, 100, 0)])
def test_merge_matches_oracle_selection(S, M, k, pad, nan):
    import bit_weight_only_quantize_b200 as q4
    vals, rows = _lists(S, M, k, seed=S * 31 + M, pad=pad, nan=nan)
    idx, val = q4.topk_merge(torch.from_numpy(vals).cuda(), torch.from_numpy(rows).cuda(), k)
    want_i, want_v = oracle.select_topk(vals.transpose(1, 0, 2).reshape(M, -1),
                                        rows.transpose(1, 0, 2).reshape(M, -1), k)
    assert np.array_equal(idx.cpu().numpy(), want_i)
    assert np.array_equal(val.cpu().numpy().astype(np.float64), want_v, equal_nan=True)


def test_merge_signed_zero_ties_by_row():
    import bit_weight_only_quantize_b200 as q4
    vals = np.array([[[-0.0, 1.0]], [[0.0, -1.0]]], dtype=np.float32)          # S=2, M=1, k=2
    rows = np.array([[[5, 9]], [[3, 11]]], dtype=np.int64)
    idx, val = q4.topk_merge(torch.from_numpy(vals).cuda(), torch.from_numpy(rows).cuda(), 2)
    assert idx.cpu().tolist() == [[9, 3]]                # -0 and +0 tie: the lower row first
    want_i, _ = oracle.select_topk(np.array([[-0.0, 1.0, 0.0, -1.0]]), np.array([[5, 9, 3, 11]]), 2)
    assert idx.cpu().numpy().tolist() == want_i.tolist()


@pytest.mark.parametrize("world,M,k", [(8, 1, 20), (3, 4, 32), (2, 1, 1)])
def test_sharded_head_emulated_on_one_gpu(world, M, k):
    import bit_weight_only_quantize_b200 as q4
    from bit_weight_only_quantize_b200.shard import shard_rows
    N, K = 60000, 2560
    W = synth_inputs.weights("outliers", N, K, seed=world)
    x = synth_inputs.activations(M, K, "bf16", seed=M)
    xf = (x.astype(np.uint32) << 16).view(np.float32)
    planted = [59999, 7, 30001, 12345]                           # in different shards, decreasing
    for i, r in enumerate(planted):
        W[r] = np.sign(xf[0]) * (0.3 - 0.02 * i)
    packed, scales, _ = oracle.quantize(W)
    dp, ds = _dev(packed, scales)
    dx = to_dev_x(x)
    li, lv = [], []
    for r in range(world):
        r0, r1 = shard_rows(N, world, r)
        i, v, _ = q4.gemv_topk(dx, dp[r0:r1], ds[r0:r1], k, row_base=r0)
        li.append(i)
        lv.append(v)
    idx, val = q4.topk_merge(torch.stack(lv), torch.stack(li), k)
    idx, val = idx.cpu().numpy(), val.cpu().numpy().astype(np.float64)
    assert idx[0, :min(k, 4)].tolist() == planted[:min(k, 4)]
    ref = oracle.matmul(x, packed, scales, threads=8)
    tol = 1e-2 * np.abs(ref).max()
    for m in range(M):
        order = np.lexsort((np.arange(N), -ref[m]))
        kth = ref[m, order[k - 1]]
        assert len(set(idx[m].tolist())) == k
        assert np.all(ref[m, idx[m]] >= kth - tol)
        assert np.all(np.abs(val[m] - ref[m, idx[m]]) <= tol)
        sure = order[:k][ref[m, order[:k]] > kth + 2 * tol]
        assert set(sure.tolist()) <= set(idx[m].tolist())


def test_sharded_head_single_process_is_the_plain_topk():
    """Without a process group the sharded head is one shard: the plain fused top-k."""
    import bit_weight_only_quantize_b200 as q4
    from bit_weight_only_quantize_b200.shard import ShardedLMHead
    packed, scales, _ = oracle.quantize(synth_inputs.weights("normal", 5000, 512, seed=1))
    head = ShardedLMHead(*_dev(packed, scales), N=5000)
    x = to_dev_x(synth_inputs.activations(2, 512, "bf16", seed=2))
    hi, hv = head.topk(x, 20)
    ti, tv, _ = q4.gemv_topk(x, *_dev(packed, scales), 20)
    assert torch.equal(hi, ti) and torch.equal(hv, tv)
