"""q4_gemv_noalloc, the decode GEMV for callers that cannot allocate device memory
(runtimes that own every device buffer, hosts that forbid allocation after
start-up, code running during a global-mode graph capture).  Called through the
C ABI, its output must match q4_gemv's (same tolerance as the split-K tests) on
consecutive calls, since every call shares the library's one scratch array.

This file is named to be collected last.  It must pass both on its own in a
fresh process and after the other tests.
"""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs
from tests._parity import rel_inf

pytestmark = pytest.mark.gpu


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("M,N,K", [(1, 1024, 2560), (4, 48, 16384), (1, 16, 8192), (1, 4096, 2560)])
def test_noalloc_matches_gemv_on_consecutive_calls(M, N, K):
    from bit_weight_only_quantize_b200 import _lib
    lib = _lib.load()
    W = synth_inputs.weights("outliers", N, K, seed=N)
    packed, scales, _ = oracle.quantize(W)
    pk = _dev(packed)
    sc = _dev(scales.view(np.int16))
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        x = _dev(synth_inputs.activations(M, K, "bf16", seed=call).view(np.int16)).view(torch.bfloat16)
        y_ref = torch.empty((M, N), dtype=torch.float32, device="cuda")
        need = lib.q4_gemv_workspace_size(M, N, K)
        ws = torch.zeros(max(need, 16), dtype=torch.uint8, device="cuda")
        _lib.check(lib.q4_gemv(x.data_ptr(), _lib.Q4_BF16, M, K, pk.data_ptr(), sc.data_ptr(), N,
                               y_ref.data_ptr(), ws.data_ptr(), ws.numel(), stream), "q4_gemv")
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        _lib.check(lib.q4_gemv_noalloc(x.data_ptr(), _lib.Q4_BF16, M, K, pk.data_ptr(), sc.data_ptr(), N,
                                       y.data_ptr(), stream), "q4_gemv_noalloc")
        torch.cuda.synchronize()
        got = y.cpu().numpy()
        assert rel_inf(got, y_ref.cpu().numpy().astype(np.float64)) <= 1e-5
        # and against the oracle itself, not only against the other entry point
        ref = oracle.matmul(synth_inputs.activations(M, K, "bf16", seed=call), packed, scales, threads=8)
        assert rel_inf(got, ref) <= 1e-5


def test_noalloc_validates_like_gemv():
    from bit_weight_only_quantize_b200 import _lib
    lib = _lib.load()
    A16 = 1 << 20
    assert lib.q4_gemv_noalloc(A16, 1, 17, 64, A16, A16, 8, A16, None) == 2
    assert lib.q4_gemv_noalloc(A16, 1, 1, 40, A16, A16, 8, A16, None) == 2
    assert lib.q4_gemv_noalloc(None, 1, 1, 64, A16, A16, 8, A16, None) == 1
    assert lib.q4_gemv_noalloc(A16 + 8, 1, 1, 64, A16, A16, 8, A16, None) == 3
    assert lib.q4_gemv_noalloc(A16, 5, 1, 64, A16, A16, 8, A16, None) == 4
