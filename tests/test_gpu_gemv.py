"""GPU parity of q4_gemv against the oracle (binary64 products of the exact dequantised
weights).  Two bars: the stated ||y - y_ref||_inf / ||y_ref||_inf tolerance (2e-3 with
f32 x, 1e-2 with bf16 x) and, tighter, the a-priori f32 summation bound per element."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs
from tests._parity import digit_path_bound, f32_sum_bound, mma_path_bound, rel_inf, to_dev_x

pytestmark = pytest.mark.gpu

TOL = {"f32": 2e-3, "bf16": 1e-2}


def gpu_gemv(x, packed, scales, workspace=None):
    import bit_weight_only_quantize_b200 as q4
    pk = torch.from_numpy(packed).cuda()
    sc = torch.from_numpy(scales.view(np.int16)).cuda()
    y = q4.gemv(to_dev_x(x), pk, sc, workspace=workspace)
    torch.cuda.synchronize()
    return y.cpu().numpy()


def roundings(K):
    # 16 products per f32x2 lane, the pair add, the scale FMA, one add per group a lane
    # owns, 4 shuffle levels and up to K/512 split partials: far below this.
    return 32 + K // 32 + 8


def check(x, W, x_dtype, tight=True):
    packed, scales, _ = oracle.quantize(W)
    y = gpu_gemv(x, packed, scales)
    ref = oracle.matmul(x, packed, scales, threads=8)
    assert y.shape == ref.shape
    err = rel_inf(y, ref)
    assert err <= TOL[x_dtype], err
    if tight:
        # the bound of the path the shape takes: M = 1 with K % 256 == 0 runs on exact
        # integer digit planes of x, M >= 2 with bf16 x and K % 256 == 0 on the bf16
        # tensor cores (exact products, f32 sums), every other shape on CUDA-core FMAs
        n, deq = roundings(W.shape[1]), oracle.dequantize(packed, scales)
        if W.shape[1] % 256 == 0 and x.shape[0] == 1:
            bound = digit_path_bound(x, deq, n)
        elif W.shape[1] % 256 == 0 and x_dtype == "bf16":
            bound = mma_path_bound(x, deq, n)
        else:
            bound = f32_sum_bound(x, deq, n)
        assert np.all(np.abs(y - ref) <= bound + 1e-30)
    return y, ref


@pytest.mark.parametrize("x_dtype", ["f32", "bf16"])
@pytest.mark.parametrize("M,N,K", [
    (1, 1, 32), (1, 17, 96), (2, 100, 2592), (3, 33, 5120), (5, 64, 1024), (8, 250, 160),
    (13, 31, 2560), (16, 100, 8192), (1, 1000, 32), (4, 16, 320),
])
def test_ragged_shapes(M, N, K, x_dtype):
    W = synth_inputs.weights("outliers", N, K, seed=M * 1000 + N)
    x = synth_inputs.activations(M, K, x_dtype, seed=M + K)
    check(x, W, x_dtype)


@pytest.mark.parametrize("M,N,K", [(1, 16, 8192), (1, 64, 4096), (4, 48, 16384), (16, 8, 2560), (1, 300, 65536)])
def test_split_k_reuses_workspace(M, N, K):
    import bit_weight_only_quantize_b200 as q4
    need = q4.gemv_workspace_size(M, N, K)
    assert need > 0, "shape expected to split K"
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    W = synth_inputs.weights("normal", N, K, seed=5)
    packed, scales, _ = oracle.quantize(W)
    ref = oracle.matmul(synth_inputs.activations(M, K, "bf16", seed=6), packed, scales, threads=8)
    for _ in range(3):                   # counters must be back at zero after each call
        x = synth_inputs.activations(M, K, "bf16", seed=6)
        y = gpu_gemv(x, packed, scales, workspace=ws)
        assert rel_inf(y, ref) <= 1e-5
    # a second input through the same workspace
    x2 = synth_inputs.activations(M, K, "bf16", seed=7)
    ref2 = oracle.matmul(x2, packed, scales, threads=8)
    assert rel_inf(gpu_gemv(x2, packed, scales, workspace=ws), ref2) <= 1e-5


def test_one_workspace_shared_across_shapes():
    """Split launches of different shapes through one workspace: the counters must
    sit where no shape's partial sums land."""
    import bit_weight_only_quantize_b200 as q4
    shapes = [(1, 2048, 2560), (1, 1024, 2560), (3, 40, 4096), (1, 16, 8192), (16, 8, 2560)]
    need = max(q4.gemv_workspace_size(*s) for s in shapes)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    cases = []
    for i, (M, N, K) in enumerate(shapes):
        W = synth_inputs.weights("normal", N, K, seed=20 + i)
        packed, scales, _ = oracle.quantize(W)
        x = synth_inputs.activations(M, K, "bf16", seed=30 + i)
        cases.append((x, packed, scales, oracle.matmul(x, packed, scales, threads=8)))
    for _ in range(2):
        for x, packed, scales, ref in cases + cases[::-1]:
            assert rel_inf(gpu_gemv(x, packed, scales, workspace=ws), ref) <= 1e-5


@pytest.mark.parametrize("M,N,K,x_dtype", [(1, 3000, 32768, "bf16"), (2, 2400, 16384, "f32"), (16, 300, 4096, "f32")])
def test_x_restaged_in_chunks(M, N, K, x_dtype):
    """K too long for one shared-memory stage of x: x is staged piecewise."""
    W = synth_inputs.weights("outliers", N, K, seed=M + N)
    x = synth_inputs.activations(M, K, x_dtype, seed=K)
    check(x, W, x_dtype, tight=False)


@pytest.mark.parametrize("x_dtype", ["bf16", "f32"])
@pytest.mark.parametrize("N,K", [(1, 256), (31, 768), (33, 2560), (1000, 5120), (4097, 256), (100000, 256),
                                 (2500, 16384), (70, 65536)])
def test_tma_path_shapes(N, K, x_dtype):
    """M = 1 with K % 256 == 0 takes the TMA kernel: ragged row blocks, idle warps
    (fewer boxes than team warps), team sizes 1..8 and K splits across blocks."""
    from bit_weight_only_quantize_b200 import _lib
    W = synth_inputs.weights("outliers", N, K, seed=N % 97 + K)
    x = synth_inputs.activations(1, K, x_dtype, seed=N)
    check(x, W, x_dtype, tight=N * K <= 2 ** 26)
    assert _lib.device_error() == 0


def test_misaligned_scales_take_generic_path():
    """Scales that are only 2-byte aligned cannot feed TMA; the generic kernel serves them."""
    import bit_weight_only_quantize_b200 as q4
    N, K = 64, 512
    W = synth_inputs.weights("normal", N, K, seed=3)
    packed, scales, _ = oracle.quantize(W)
    x = synth_inputs.activations(1, K, "bf16", seed=3)
    sc_store = torch.zeros(N * K // 32 + 8, dtype=torch.int16, device="cuda")
    sc = sc_store[1:1 + N * K // 32].view(N, K // 32)
    sc.copy_(torch.from_numpy(scales.view(np.int16)))
    y = q4.gemv(to_dev_x(x), torch.from_numpy(packed).cuda(), sc)
    torch.cuda.synchronize()
    assert rel_inf(y.cpu().numpy(), oracle.matmul(x, packed, scales)) <= 1e-5


def test_too_small_workspace_rejected():
    import bit_weight_only_quantize_b200 as q4
    M, N, K = 1, 16, 32768
    assert q4.gemv_workspace_size(M, N, K) > 16      # the shape splits K
    ws = torch.zeros(16, dtype=torch.uint8, device="cuda")
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    pk = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    sc = torch.zeros((N, K // 32), dtype=torch.int16, device="cuda")
    with pytest.raises(q4.Q4Error):
        q4.gemv(x, pk, sc, workspace=ws)


def test_zero_rows_and_zero_groups_exact():
    W = synth_inputs.weights("normal", 64, 2560, seed=8)
    W[5] = 0.0
    W[9, 64:96] = 0.0
    x = synth_inputs.activations(2, 2560, "bf16", seed=8)
    y, ref = check(x, W, "bf16")
    assert np.all(y[:, 5] == 0.0)


@pytest.mark.parametrize("w", [synth_inputs.DECODE_SMALL, *synth_inputs.DECODE_PROJ, *synth_inputs.SMALL_BATCH],
                         ids=lambda w: w.name)
def test_config_shapes(w):
    W, x = synth_inputs.make(w, seed=0)
    check(x, W, w.x_dtype, tight=w.N * w.K <= 4096 * 2560 and w.M <= 4)


def test_lm_head_full():
    w = synth_inputs.LM_HEAD
    W, x = synth_inputs.make(w, seed=0)
    check(x, W, w.x_dtype, tight=False)


def test_empty_shapes():
    import bit_weight_only_quantize_b200 as q4
    x = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    pk = torch.zeros((8, 32), dtype=torch.uint8, device="cuda")
    sc = torch.zeros((8, 2), dtype=torch.int16, device="cuda")
    assert q4.gemv(x, pk, sc).shape == (0, 8)
    x = torch.zeros((2, 64), dtype=torch.bfloat16, device="cuda")
    assert q4.gemv(x, pk[:0], sc[:0]).shape == (2, 0)
