"""Pins for the oracle's greedy LM-head step: index and value of the largest logit of
y = x . dequant(W)^T, lowest index on ties.  Checked on planted winners, exact ties and
against the oracle's own logits."""
import numpy as np

import oracle
import synth_inputs


def _q(W):
    packed, scales, _ = oracle.quantize(W)
    return packed, scales


def test_planted_winner_per_row():
    K, N, M = 256, 300, 3
    W = synth_inputs.weights("normal", N, K, seed=1)
    x = synth_inputs.activations(M, K, "f32", seed=2)
    winners = [17, 250, 0]
    for m, r in enumerate(winners):
        W[r] = np.sign(x[m]) * 0.5                     # aligned with x row m: a far larger logit
    packed, scales = _q(W)
    idx, val = oracle.argmax(x, packed, scales)
    assert idx.tolist() == winners
    y = oracle.matmul(x, packed, scales)
    assert np.array_equal(val, y[np.arange(M), idx])


def test_ties_take_the_lowest_index():
    K, N = 64, 10
    W = synth_inputs.weights("normal", N, K, seed=3) * 0.1
    x = np.ones((1, K), dtype=np.float32)
    W[7] = 0.3
    W[4] = 0.3                                          # identical rows 4 and 7: equal logits
    packed, scales = _q(W)
    idx, val = oracle.argmax(x, packed, scales)
    assert idx[0] == 4
    assert val[0] == oracle.matmul(x, packed, scales)[0, 7]


def test_matches_logits_max():
    K, N, M = 512, 1000, 4
    packed, scales = _q(synth_inputs.weights("outliers", N, K, seed=4))
    x = synth_inputs.activations(M, K, "bf16", seed=5)
    idx, val = oracle.argmax(x, packed, scales, threads=4)
    y = oracle.matmul(x, packed, scales, threads=4)
    assert np.array_equal(val, y.max(axis=1))
    for m in range(M):
        assert np.all(y[m, :idx[m]] < val[m])           # nothing before the index reaches the max
