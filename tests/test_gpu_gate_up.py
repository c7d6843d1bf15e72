"""GPU parity of q4_gemv_gate_up: y = silu(x . dequant(Wg)^T) * (x . dequant(Wu)^T) in one
launch, against the oracle's binary64 gate_up."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs
from tests._parity import rel_inf, to_dev_x

pytestmark = pytest.mark.gpu

TOL = {"f32": 2e-3, "bf16": 1e-2}


def _pair(N, K, seed, kind="outliers"):
    out = []
    for i in range(2):
        packed, scales, _ = oracle.quantize(synth_inputs.weights(kind, N, K, seed=seed + i))
        out.append((packed, scales))
    return out


def _dev(m):
    return torch.from_numpy(m[0]).cuda(), torch.from_numpy(m[1].view(np.int16)).cuda()


def run(M, N, K, x_dtype, seed, static=False, kind="outliers"):
    import bit_weight_only_quantize_b200 as q4
    gate, up = _pair(N, K, seed, kind)
    x = synth_inputs.activations(M, K, x_dtype, seed=seed + 7)
    y = q4.gemv_gate_up(to_dev_x(x), _dev(gate), _dev(up), weights_static=static)
    torch.cuda.synchronize()
    ref = oracle.gate_up(x, gate, up, threads=8)
    err = rel_inf(y.cpu().numpy(), ref)
    assert err <= TOL[x_dtype], err
    return y, ref


@pytest.mark.parametrize("x_dtype", ["f32", "bf16"])
def test_decode_mlp_shape(x_dtype):
    # QORA-4B-shaped MLP decode step: K = 2560 hidden, N = 4096 intermediate rows per matrix
    run(1, 4096, 2560, x_dtype, seed=1)


@pytest.mark.parametrize("M,N,K", [(1, 100, 512), (3, 33, 2560), (8, 250, 256), (16, 64, 1024), (2, 1, 768)])
def test_ragged_shapes(M, N, K):
    run(M, N, K, "bf16", seed=M * 100 + N, static=(M % 2 == 0))


def test_student_t_weights_small_batch():
    run(4, 4096, 2560, "bf16", seed=5, kind="student_t")


def test_zero_gate_rows_give_zero():
    import bit_weight_only_quantize_b200 as q4
    N, K = 48, 512
    gate, up = _pair(N, K, seed=9)
    gp = gate[0].copy()
    gp[::3] = 0x88                         # codes 8: gate weight 0 -> silu(0) = 0
    x = synth_inputs.activations(1, K, "bf16", seed=3)
    y = q4.gemv_gate_up(to_dev_x(x), _dev((gp, gate[1])), _dev(up)).cpu().numpy()
    assert np.all(y[:, ::3] == 0.0)


def test_unsupported_k_is_rejected():
    import bit_weight_only_quantize_b200 as q4
    N, K = 16, 96                          # K % 256 != 0
    gate, up = _pair(N, K, seed=2)
    x = to_dev_x(synth_inputs.activations(1, K, "bf16", seed=1))
    with pytest.raises(q4.Q4Error):
        q4.gemv_gate_up(x, _dev(gate), _dev(up))
