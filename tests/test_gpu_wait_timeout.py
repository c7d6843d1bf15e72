"""Failure detection without a GPU fault: every wait of the TMA GEMV kernels is bounded,
and a wait that runs out is reported through the library's device error word while the
kernel drains its own transfers and returns.  q4_set_consumer_wait_limit(0) makes each
launch give up at its first wait (the drain keeps its 1 s limit, so no transfer is left
in flight when a block exits).  The tests check that the timeout is reported, that the
workspace is left as a completed call leaves it (zero at rest), and that the next normal
call on the same workspace matches the oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs
from tests._parity import rel_inf, to_dev_x

pytestmark = pytest.mark.gpu

WAIT_TIMEOUT = 1          # Q4_DEVICE_ERR_WAIT_TIMEOUT
DEFAULT_LIMIT_NS = 10 ** 9


def _weights(N, K, seed):
    W = synth_inputs.weights("normal", N, K, seed=seed)
    packed, scales, _ = oracle.quantize(W)
    return packed, scales, torch.from_numpy(packed).cuda(), torch.from_numpy(scales.view(np.int16)).cuda()


class _GiveUpAtFirstWait:
    def __enter__(self):
        from bit_weight_only_quantize_b200 import _lib
        self.lib = _lib.load()
        self.prev = self.lib.q4_set_consumer_wait_limit(0)
        return self

    def __exit__(self, *exc):
        torch.cuda.synchronize()
        self.lib.q4_set_consumer_wait_limit(self.prev)


@pytest.mark.parametrize("M,N,K,x_dtype", [(1, 16, 8192, "bf16"), (1, 4096, 2560, "bf16"), (4, 48, 16384, "bf16"),
                                           (1, 300, 4096, "f32")])
def test_gemv_timeout_reported_then_recovers(M, N, K, x_dtype):
    import bit_weight_only_quantize_b200 as q4
    from bit_weight_only_quantize_b200 import _lib
    packed, scales, pk, sc = _weights(N, K, seed=N + K)
    x = synth_inputs.activations(M, K, x_dtype, seed=M)
    xd = to_dev_x(x)
    need = q4.gemv_workspace_size(M, N, K)
    ws = torch.zeros(max(need, 16), dtype=torch.uint8, device="cuda")
    assert _lib.device_error() in (0, WAIT_TIMEOUT)          # start from a clear word
    assert _lib.device_error() == 0
    with _GiveUpAtFirstWait() as g:
        q4.gemv(xd, pk, sc, workspace=ws)
    assert g.prev == DEFAULT_LIMIT_NS
    assert _lib.device_error() == WAIT_TIMEOUT                 # reported (and cleared)
    assert int(torch.count_nonzero(ws[:4096])) == 0            # split-K counters back at zero
    y = q4.gemv(xd, pk, sc, workspace=ws)
    torch.cuda.synchronize()
    assert _lib.device_error() == 0
    assert rel_inf(y.cpu().numpy(), oracle.matmul(x, packed, scales, threads=8)) <= 1e-5
    assert int(torch.count_nonzero(ws[:4096])) == 0


def test_topk_timeout_leaves_workspace_at_rest():
    import bit_weight_only_quantize_b200 as q4
    from bit_weight_only_quantize_b200 import _lib
    N, K, k = 5000, 2560, 20
    packed, scales, pk, sc = _weights(N, K, seed=3)
    x = synth_inputs.activations(1, K, "bf16", seed=4)
    xd = to_dev_x(x)
    ws = torch.zeros(max(16, q4.gemv_topk_workspace_size(1, N, K, k)), dtype=torch.uint8, device="cuda")
    _lib.device_error()
    with _GiveUpAtFirstWait():
        q4.gemv_topk(xd, pk, sc, k, workspace=ws)
    assert _lib.device_error() == WAIT_TIMEOUT
    assert int(torch.count_nonzero(ws[:16])) == 0              # block counter and published bar
    idx, val, _ = q4.gemv_topk(xd, pk, sc, k, workspace=ws)
    torch.cuda.synchronize()
    assert _lib.device_error() == 0
    ref_idx, ref_val = oracle.topk(x, packed, scales, k, threads=8)
    assert idx.cpu().numpy()[0, 0] == ref_idx[0, 0]
    assert np.max(np.abs(val.cpu().numpy() - ref_val)) <= 1e-5 * np.max(np.abs(ref_val))
