"""GPU parity of q4_gemm (tcgen05 tensor cores) against the oracle.

Bars: ||y - y_ref||_inf / ||y_ref||_inf <= 1e-2 (bf16 activations and output), and per
element the bound that follows from the arithmetic: each weight rounded once to bf16
(relative error <= 2^-8), exact bf16 products, f32 accumulation over K terms, one
rounding of the result to bf16:
    |y - y_ref| <= 2^-8 |y_ref| + (2^-8 + K 2^-22) sum_k |x_k w'_k|   (x 1.1 slack).
Large shapes compare a sample of rows and columns the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs
from tests._parity import rel_inf

pytestmark = pytest.mark.gpu


def bf16_bits_to_f64(b):
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def run_gemm(x_bits, packed, scales):
    import bit_weight_only_quantize_b200 as q4
    from bit_weight_only_quantize_b200 import _lib
    x = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).cuda()
    y = q4.gemm(x, torch.from_numpy(packed).cuda(), torch.from_numpy(scales.view(np.int16)).cuda())
    torch.cuda.synchronize()
    assert _lib.device_error() == 0        # no bounded wait ran out
    return bf16_bits_to_f64(y.view(torch.int16).cpu().numpy().view(np.uint16))


def check(M, N, K, kind="normal", seed=0, m_sample=None, n_sample=None):
    W = synth_inputs.weights(kind, N, K, seed=seed)
    packed, scales, _ = oracle.quantize(W)
    x = synth_inputs.activations(M, K, "bf16", seed=seed + 1)
    y = run_gemm(x, packed, scales)
    assert y.shape == (M, N)
    rows = np.arange(M) if m_sample is None else np.unique(np.linspace(0, M - 1, m_sample).astype(np.int64))
    cols = np.arange(N) if n_sample is None else np.unique(np.linspace(0, N - 1, n_sample).astype(np.int64))
    xs = np.ascontiguousarray(x[rows])
    ref = oracle.matmul(xs, packed, scales, rows=cols, threads=8)
    got = y[np.ix_(rows, cols)]
    assert rel_inf(got, ref) <= 1e-2
    wd = oracle.dequantize(packed[cols], scales[cols])
    mag = np.abs(bf16_bits_to_f64(xs)) @ np.abs(wd).T
    bound = 1.1 * (2.0 ** -8 * np.abs(ref) + (2.0 ** -8 + K * 2.0 ** -22) * mag)
    assert np.all(np.abs(got - ref) <= bound + 1e-30)
    return y


@pytest.mark.parametrize("M,N,K", [
    (1, 16, 32), (130, 72, 96), (300, 200, 2560), (513, 1000, 1024), (64, 75, 256), (129, 129, 160),
])
def test_small_and_ragged(M, N, K):
    check(M, N, K, kind="outliers", seed=M + N)


def test_tile_256x128():
    # enough 256 x 128 tiles to fill every SM: two 128-row accumulators per tile
    check(2048, 4096, 256, seed=3, m_sample=96, n_sample=96)


def test_tile_128x128():
    check(1024, 2560, 512, seed=4, m_sample=96, n_sample=96)


@pytest.mark.parametrize("M,N,K", [
    (2048, 2432, 128),     # 8 x 10 CTA-pair tiles of 256 x 256, ragged in N
    (512, 2048, 256),      # 2 x 16 pair tiles of 256 x 128 (K too short to split)
    (2176, 4160, 64),      # 9 x 17 = 153 pair tiles: pairs run two or three tiles each, ragged M and N
])
def test_large_tiles_full_output(M, N, K):
    """Every output element of the large-tile paths against the oracle (not a sample)."""
    check(M, N, K, kind="outliers", seed=M + K)


@pytest.mark.parametrize("M,N,K", [
    (300, 200, 2560),      # 2 pair tiles, 2 pairs per tile (40 k-blocks: 20 each)
    (260, 130, 1088),      # 2 pairs per tile over 17 k-blocks (8, 9), ragged M and N
    (768, 2048, 512),      # 24 pair tiles, 2 pairs per tile (8 k-blocks: 4 each)
    (700, 2000, 640),      # 24 pair tiles, 2 pairs per tile, ragged M and N
])
def test_split_k_clusters_full_output(M, N, K):
    """Pair tiles whose K range is split over the 2 CTA pairs of one cluster, the partial
    slices exchanged through distributed shared memory: every output element."""
    check(M, N, K, kind="outliers", seed=M + N + K)


def test_split_k_clusters_repeatable():
    """The split partials are summed in a fixed order: two runs agree bit for bit."""
    W = synth_inputs.weights("normal", 512, 2560, seed=5)
    packed, scales, _ = oracle.quantize(W)
    x = synth_inputs.activations(512, 2560, "bf16", seed=6)
    assert np.array_equal(run_gemm(x, packed, scales), run_gemm(x, packed, scales))


def test_zero_weights_give_zero():
    M, N, K = 256, 64, 512
    W = np.zeros((N, K), np.float32)
    packed, scales, _ = oracle.quantize(W)
    x = synth_inputs.activations(M, K, "bf16", seed=9)
    assert np.all(run_gemm(x, packed, scales) == 0.0)


@pytest.mark.parametrize("w", synth_inputs.PREFILL, ids=lambda w: w.name)
def test_prefill_configs(w):
    check(w.M, w.N, w.K, kind=w.weights, seed=0, m_sample=64, n_sample=64)


def test_empty_and_device_error():
    import bit_weight_only_quantize_b200 as q4
    from bit_weight_only_quantize_b200 import _lib
    x = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    pk = torch.zeros((8, 32), dtype=torch.uint8, device="cuda")
    sc = torch.zeros((8, 2), dtype=torch.int16, device="cuda")
    assert q4.gemm(x, pk, sc).shape == (0, 8)
    assert _lib.device_error() == 0
