"""GPU parity of the INT8 weight path (the INT8 layers of a mixed INT8/INT4 model) against
the oracle: q4_int8_quantize bit-exact (codes, scales, flags), q4_int8_gemv within the
GEMV tolerance (2e-3 with f32 x, 1e-2 with bf16 x, relative to the largest |y|)."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs
from tests._parity import digit_path_bound, f32_sum_bound, rel_inf, to_dev_x

pytestmark = pytest.mark.gpu

TOL = {"f32": 2e-3, "bf16": 1e-2}


def _quantize_dev(W):
    import bit_weight_only_quantize_b200 as q4
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    codes, scales = q4.int8_quantize(torch.from_numpy(W).cuda(), flags=flags)
    torch.cuda.synchronize()
    return codes, scales, int(flags.item())


@pytest.mark.parametrize("kind,N,K", [("outliers", 256, 2560), ("normal", 1000, 96), ("student_t", 33, 32),
                                      ("normal", 4096, 2560)])
def test_quantize_bit_exact(kind, N, K):
    W = synth_inputs.weights(kind, N, K, seed=N + K)
    codes, scales, flags = _quantize_dev(W)
    want_c, want_s, want_f = oracle.quantize8(W)
    assert np.array_equal(codes.cpu().numpy(), want_c)
    assert np.array_equal(scales.cpu().numpy().view(np.uint16), want_s)
    assert flags == want_f


def test_quantize_special_groups():
    W = synth_inputs.weights("normal", 4, 128, seed=6)
    W[0, 32:64] = 0.0                                       # zero group
    W[1, 5] = np.inf                                        # non-finite
    W[2, 64:96] = 1.0e7                                     # scale overflows binary16
    a = np.float32(127 * 1.4 * 2.0 ** -24)                  # subnormal scale rounded down: clamp at -128
    W[3, 96:128] = 0.0
    W[3, 96], W[3, 97] = -a, a
    codes, scales, flags = _quantize_dev(W)
    want_c, want_s, want_f = oracle.quantize8(W)
    assert np.array_equal(codes.cpu().numpy(), want_c)
    assert np.array_equal(scales.cpu().numpy().view(np.uint16), want_s)
    assert flags == want_f == 3
    assert want_c[3, 96] == -128 and want_c[3, 97] == 127


@pytest.mark.parametrize("M,N,K,x_dtype", [(1, 4096, 2560, "f32"), (1, 4096, 2560, "bf16"), (4, 1000, 1024, "bf16"),
                                           (16, 333, 256, "bf16"), (3, 50, 96, "f32"), (2, 7, 32, "bf16"),
                                           # more rows than the grid holds warps: rows are walked in rounds
                                           (1, 20000, 2560, "bf16"),
                                           # 160 KB of f32 x in shared memory: one block per SM
                                           (16, 300, 2560, "f32")])
def test_gemv_matches_oracle(M, N, K, x_dtype):
    import bit_weight_only_quantize_b200 as q4
    codes, scales, _ = oracle.quantize8(synth_inputs.weights("outliers", N, K, seed=M * 7 + N))
    x = synth_inputs.activations(M, K, x_dtype, seed=M)
    y = q4.int8_gemv(to_dev_x(x), torch.from_numpy(codes).cuda(), torch.from_numpy(scales.view(np.int16)).cuda())
    torch.cuda.synchronize()
    got = y.cpu().numpy()
    ref = oracle.matmul8(x, codes, scales, threads=8)
    err = rel_inf(got, ref)
    assert err <= TOL[x_dtype], err
    assert np.all(np.abs(got - ref) <= int8_bound(x, codes, scales) + 1e-30)


def int8_bound(x, codes, scales):
    """Per-element bound of the path the shape takes.  M = 1 with K % 256 == 0: the
    digit-plane path (x rounded per group of 32, exact integer group sums, one rounding
    combining two planes, the scale FMA and the f32 accumulation per plane).  Otherwise:
    exact code x exact x products summed in f32 (16 per block of k, one scale FMA per
    block, a lane's blocks, the warp's 5 shuffle adds)."""
    M, K = x.shape
    deq = oracle.dequantize8(codes, scales)
    if M == 1 and K % 256 == 0:
        return digit_path_bound(x, deq, 2 * (K // 32) + 40)
    return f32_sum_bound(x, deq, 16 + K // 16 + 8)


@pytest.mark.parametrize("N,x_dtype", [(4096, "bf16"), (33, "f32"), (20000, "bf16"), (1, "bf16")])
def test_gemv_tma_path_k_large(N, x_dtype):
    """M = 1, K % 256 == 0: the TMA kernel's integer path, K = 2560 and K = 8192."""
    import bit_weight_only_quantize_b200 as q4
    for K in (2560, 8192):
        codes, scales, _ = oracle.quantize8(synth_inputs.weights("outliers", N, K, seed=N + K))
        x = synth_inputs.activations(1, K, x_dtype, seed=K)
        y = q4.int8_gemv(to_dev_x(x), torch.from_numpy(codes).cuda(), torch.from_numpy(scales.view(np.int16)).cuda())
        torch.cuda.synchronize()
        got, ref = y.cpu().numpy(), oracle.matmul8(x, codes, scales, threads=8)
        assert rel_inf(got, ref) <= 1e-5
        assert np.all(np.abs(got - ref) <= int8_bound(x, codes, scales) + 1e-30)


def _mixed_case(M, K, spec, x_dtype, seed):
    """Matrices [(N, bits)] quantised by the oracle, on the device."""
    import bit_weight_only_quantize_b200 as q4
    host, dev = [], []
    for i, (n, bits) in enumerate(spec):
        W = synth_inputs.weights("outliers", n, K, seed=seed + i)
        codes, scales, _ = (oracle.quantize8 if bits == 8 else oracle.quantize)(W)
        host.append((codes, scales, bits))
        dev.append((torch.from_numpy(codes).cuda(), torch.from_numpy(scales.view(np.int16)).cuda(), bits))
    x = synth_inputs.activations(M, K, x_dtype, seed=seed)
    ys = q4.gemv_mixed(to_dev_x(x), dev)
    torch.cuda.synchronize()
    for (codes, scales, bits), y in zip(host, ys):
        got = y.cpu().numpy()
        if bits == 8:
            ref = oracle.matmul8(x, codes, scales, threads=8)
            bound = int8_bound(x, codes, scales)
        else:
            ref = oracle.matmul(x, codes, scales, threads=8)
            bound = None
            if M == 1 and K % 256 == 0:
                bound = digit_path_bound(x, oracle.dequantize(codes, scales), 2 * (K // 32) + 40)
        assert rel_inf(got, ref) <= 1e-5, bits
        if bound is not None:
            assert np.all(np.abs(got - ref) <= bound + 1e-30)


@pytest.mark.parametrize("spec", [
    [(2048, 4), (1024, 8), (4096, 4)],          # attention INT8 beside Q4 projections, one launch
    [(4096, 8), (4096, 8)],                      # INT8 only
    [(33, 8), (17, 4), (0, 8), (300, 8)],        # ragged row blocks, an empty matrix
    [(16, 8), (16, 4)],                          # skinny: K split across blocks
])
def test_mixed_single_launch(spec):
    _mixed_case(1, 2560, spec, "bf16", seed=len(spec))
    _mixed_case(1, 8192, spec, "f32", seed=7)


@pytest.mark.parametrize("M,K", [(3, 2560), (1, 96), (16, 512)])
def test_mixed_separate_launches(M, K):
    """Shapes the single launch does not take: Q4 in one launch, each INT8 matrix in its own."""
    _mixed_case(M, K, [(1000, 8), (500, 4), (64, 8)], "bf16", seed=M + K)


def test_gemv_x_too_large_is_rejected():
    import bit_weight_only_quantize_b200 as q4
    K = 8192                                               # 16 x rows of f32 x: 512 KB of shared memory
    codes = torch.zeros((8, K), dtype=torch.int8, device="cuda")
    scales = torch.zeros((8, K // 32), dtype=torch.int16, device="cuda")
    x = torch.zeros((16, K), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(q4.Q4Error):
        q4.int8_gemv(x, codes, scales)
