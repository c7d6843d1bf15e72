"""Pins for the oracle's top-k selection of LM-head logits: the k largest logits of
y = x . dequant(W)^T per x row, larger first, the lower row among equal values, a NaN
above every number; rows past the candidates hold index -1 and value NaN.

Checked against a brute force written with Python's ``sorted`` on (value, row) tuples,
against the oracle's greedy argmax for k = 1, and on planted winners, exact ties, short
lists, NaN candidates and shard offsets."""
import math

import numpy as np
import pytest

import oracle
import synth_inputs


def _q(W):
    packed, scales, _ = oracle.quantize(W)
    return packed, scales


def _brute(values, rows, k):
    out = []
    for vr, ir in zip(values.tolist(), rows.tolist()):
        best = sorted([(v, i) for v, i in zip(vr, ir) if i >= 0], key=lambda t: (0 if math.isnan(t[0]) else 1,
                                                  0.0 if math.isnan(t[0]) else -t[0], t[1]))[:k]
        best += [(math.nan, -1)] * (k - len(best))
        out.append(best)
    return out


def _same(got_i, got_v, want):
    for m, row in enumerate(want):
        assert got_i[m].tolist() == [r for _, r in row]
        for gv, (wv, _) in zip(got_v[m].tolist(), row):
            assert (math.isnan(gv) and math.isnan(wv)) or gv == wv


@pytest.mark.parametrize("M,N,K,k", [(1, 300, 64, 20), (3, 50, 96, 7), (2, 33, 256, 32), (4, 5, 32, 20)])
def test_matches_brute_force(M, N, K, k):
    packed, scales = _q(synth_inputs.weights("outliers", N, K, seed=N))
    x = synth_inputs.activations(M, K, "bf16", seed=M)
    idx, val = oracle.topk(x, packed, scales, k)
    y = oracle.matmul(x, packed, scales)
    _same(idx, val, _brute(y, np.broadcast_to(np.arange(N), y.shape), k))


def test_k1_is_the_greedy_argmax():
    packed, scales = _q(synth_inputs.weights("normal", 700, 256, seed=3))
    x = synth_inputs.activations(5, 256, "bf16", seed=4)
    idx, val = oracle.topk(x, packed, scales, 1)
    ai, av = oracle.argmax(x, packed, scales)
    assert np.array_equal(idx[:, 0], ai) and np.array_equal(val[:, 0], av)


def test_planted_winners_in_order():
    K, N = 128, 400
    W = synth_inputs.weights("normal", N, K, seed=5) * 0.05
    x = np.ones((1, K), dtype=np.float32)
    planted = [311, 2, 150, 399]                   # descending planted logits 4c, 3c, 2c, c
    for i, r in enumerate(planted):
        W[r] = 0.25 * (len(planted) - i)
    idx, val = oracle.topk(x, *_q(W), 4)
    assert idx[0].tolist() == planted
    assert np.all(np.diff(val[0]) < 0)


def test_ties_take_lower_rows_first():
    K, N = 64, 12
    W = synth_inputs.weights("normal", N, K, seed=6) * 0.01
    x = np.ones((1, K), dtype=np.float32)
    for r in (9, 3, 6):
        W[r] = 0.3                                 # three identical best rows
    idx, val = oracle.topk(x, *_q(W), 4)
    assert idx[0, :3].tolist() == [3, 6, 9]
    assert val[0, 0] == val[0, 1] == val[0, 2] > val[0, 3]


def test_short_list_pads_and_row_base_offsets():
    packed, scales = _q(synth_inputs.weights("normal", 3, 64, seed=7))
    x = synth_inputs.activations(2, 64, "f32", seed=8)
    idx, val = oracle.topk(x, packed, scales, 5, row_base=1000)
    assert np.all(idx[:, 3:] == -1) and np.all(np.isnan(val[:, 3:]))
    assert sorted(idx[0, :3].tolist()) == [1000, 1001, 1002]
    i0, v0 = oracle.topk(x, packed, scales, 5)
    assert np.array_equal(idx[:, :3], i0[:, :3] + 1000) and np.array_equal(val[:, :3], v0[:, :3])


def test_nan_ranks_first_and_merge_of_shards():
    vals = np.array([[1.0, np.nan, 3.0, -2.0, 3.0, np.nan]])
    rows = np.array([[10, 11, 12, 13, 14, 15]])
    idx, val = oracle.select_topk(vals, rows, 4)
    assert idx[0].tolist() == [11, 15, 12, 14]
    _same(idx, val, _brute(vals, rows, 4))
    # padding (negative index, NaN value) takes no place, even though a NaN ranks first
    pad = np.array([[np.nan, 2.0, np.nan, 5.0]]), np.array([[-1, 40, -1, 41]])
    idx, val = oracle.select_topk(*pad, 3)
    assert idx[0].tolist() == [41, 40, -1] and np.isnan(val[0, 2])
    _same(idx, val, _brute(*pad, 3))
    # selection over the union of two shards' lists equals selection over all logits
    rng = np.random.default_rng(9)
    y = rng.standard_normal((3, 200))
    y[:, 50] = y[:, 150]                           # a tie across the shard boundary
    full_i, full_v = oracle.select_topk(y, np.broadcast_to(np.arange(200), y.shape), 20)
    parts = [oracle.select_topk(y[:, s:s + 100], np.broadcast_to(np.arange(s, s + 100), (3, 100)), 20)
             for s in (0, 100)]
    mi, mv = oracle.select_topk(np.concatenate([p[1] for p in parts], 1),
                                np.concatenate([p[0] for p in parts], 1), 20)
    assert np.array_equal(mi, full_i) and np.array_equal(mv, full_v)
