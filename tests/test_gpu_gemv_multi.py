"""GPU parity of q4_gemv_multi (several weight matrices sharing x in one launch)."""
import numpy as np
import pytest
import torch

import oracle
import synth_inputs
from tests._parity import rel_inf, to_dev_x

pytestmark = pytest.mark.gpu


def _prep(Ns, K, kind="outliers", seed=0):
    mats = []
    for i, n in enumerate(Ns):
        W = synth_inputs.weights(kind, n, K, seed=seed + i)
        packed, scales, _ = oracle.quantize(W)
        mats.append((packed, scales))
    return mats


def _dev(mats):
    return [(torch.from_numpy(p).cuda(), torch.from_numpy(s.view(np.int16)).cuda()) for p, s in mats]


@pytest.mark.parametrize("static", [False, True])
@pytest.mark.parametrize("M,x_dtype", [(1, "bf16"), (1, "f32"), (4, "bf16"), (16, "bf16")])
def test_decode_projections(M, x_dtype, static):
    import bit_weight_only_quantize_b200 as q4
    Ns, K = [2048, 4096, 1024], 2560
    mats = _prep(Ns, K)
    x = synth_inputs.activations(M, K, x_dtype, seed=M)
    ys = q4.gemv_multi(to_dev_x(x), _dev(mats), weights_static=static)
    torch.cuda.synchronize()
    for (packed, scales), y in zip(mats, ys):
        ref = oracle.matmul(x, packed, scales, threads=8)
        assert rel_inf(y.cpu().numpy(), ref) <= 1e-5


@pytest.mark.parametrize("Ns,K", [([17, 0, 300, 5], 512), ([1, 2, 3, 4], 256), ([100, 70], 96), ([4000, 33], 8192)])
def test_ragged_and_empty(Ns, K):
    import bit_weight_only_quantize_b200 as q4
    mats = _prep(Ns, K, seed=7)
    x = synth_inputs.activations(2, K, "bf16", seed=3)
    ys = q4.gemv_multi(to_dev_x(x), _dev(mats))
    torch.cuda.synchronize()
    for (packed, scales), y, n in zip(mats, ys, Ns):
        assert y.shape == (2, n)
        if n:
            assert rel_inf(y.cpu().numpy(), oracle.matmul(x, packed, scales)) <= 1e-5


def test_matches_single_calls():
    import bit_weight_only_quantize_b200 as q4
    Ns, K = [512, 96, 1024], 1024
    mats = _prep(Ns, K, seed=11)
    xd = to_dev_x(synth_inputs.activations(1, K, "bf16", seed=5))
    dm = _dev(mats)
    ys = q4.gemv_multi(xd, dm)
    for (pk, sc), y in zip(dm, ys):
        y1 = q4.gemv(xd, pk, sc)
        torch.cuda.synchronize()
        assert rel_inf(y.cpu().numpy(), y1.cpu().numpy().astype(np.float64)) <= 1e-6


def test_graph_chain_with_static_weights():
    """Dependent launches captured in a graph, each allowed to stream its weights
    before its predecessor ends; x is rewritten between steps by a copy kernel."""
    import bit_weight_only_quantize_b200 as q4
    Ns, K = [2048, 4096, 1024], 2560
    mats = _prep(Ns, K, seed=21)
    dm = _dev(mats)
    xs = [synth_inputs.activations(1, K, "bf16", seed=40 + i) for i in range(4)]
    xsrc = [to_dev_x(x) for x in xs]
    xd = torch.empty_like(xsrc[0])
    outs = [[torch.empty((1, n), dtype=torch.float32, device="cuda") for n in Ns] for _ in xs]
    need = q4.gemv_multi_workspace_size(1, K, Ns)
    ws = torch.zeros(max(need, 16), dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        q4.gemv_multi(xd, dm, outs[0], ws, weights_static=True)       # warm-up outside the capture
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            for i in range(len(xs)):
                xd.copy_(xsrc[i])
                q4.gemv_multi(xd, dm, outs[i], ws, weights_static=True)
    g.replay()
    torch.cuda.synchronize()
    for i, x in enumerate(xs):
        for (packed, scales), y in zip(mats, outs[i]):
            assert rel_inf(y.cpu().numpy(), oracle.matmul(x, packed, scales, threads=8)) <= 1e-5


@pytest.mark.parametrize("M,x_dtype", [(1, "bf16"), (1, "f32"), (3, "bf16")])
def test_prepared_call_matches_gemv_multi(M, x_dtype):
    """GemvMulti checks the weights once and launches the same kernel: identical bits."""
    import bit_weight_only_quantize_b200 as q4
    Ns, K = [2048, 4096, 1024], 2560
    dm = _dev(_prep(Ns, K, seed=21))
    plan = q4.GemvMulti(dm, M, K, torch.float32 if x_dtype == "f32" else torch.bfloat16, weights_static=True)
    for seed in (1, 2):
        x = synth_inputs.activations(M, K, x_dtype, seed=seed)
        xd = to_dev_x(x)
        ys = [y.clone() for y in plan(xd)]
        ref = q4.gemv_multi(xd, dm)
        torch.cuda.synchronize()
        for y, r, (p, s) in zip(ys, ref, _prep(Ns, K, seed=21)):
            assert torch.equal(y, r)
            assert rel_inf(y.cpu().numpy(), oracle.matmul(x, p, s, threads=8)) <= (2e-3 if x_dtype == "f32" else 1e-2)
    with pytest.raises(ValueError):
        plan(to_dev_x(synth_inputs.activations(M + 1, K, x_dtype, seed=3)))      # wrong shape
    with pytest.raises(TypeError):
        plan(torch.zeros((M, K), dtype=torch.float16, device="cuda"))            # wrong dtype


@pytest.mark.parametrize("M,x_dtype,shared", [(1, "bf16", True), (1, "f32", False), (4, "bf16", False)])
def test_host_step_graph_matches_oracle(M, x_dtype, shared):
    """GemvMulti.host_step: pinned x in, the GEMVs, outputs to pinned host memory, as one
    graph; replayed with new host inputs it gives the prepared call's bits each time."""
    import bit_weight_only_quantize_b200 as q4
    Ns, K = [2048, 4096, 1024], 2560
    mats = _prep(Ns, K, seed=31)
    dm = _dev(mats)
    dt = torch.float32 if x_dtype == "f32" else torch.bfloat16
    if shared:                                        # M == 1: outputs are views of one buffer
        y_dev = torch.empty((M, sum(Ns)), dtype=torch.float32, device="cuda")
        outs = [y_dev[:, a:a + n] for a, n in zip(np.cumsum([0] + Ns[:-1]).tolist(), Ns)]
    else:
        y_dev, outs = None, None
    plan = q4.GemvMulti(dm, M, K, dt, outs=outs, weights_static=True)
    x_host = torch.empty((M, K), dtype=dt).pin_memory()
    if shared:
        y_host = torch.empty_like(y_dev, device="cpu").pin_memory()
    else:
        y_host = [torch.empty((M, n), dtype=torch.float32).pin_memory() for n in Ns]
    step = plan.host_step(x_host, y_host, y_dev=y_dev)
    for seed in (4, 5):
        x = synth_inputs.activations(M, K, x_dtype, seed=seed)
        x_host.copy_(torch.from_numpy(x.view(np.int16)).view(torch.bfloat16) if x_dtype == "bf16"
                     else torch.from_numpy(x))
        step()
        torch.cuda.synchronize()
        got = torch.split(y_host, Ns, dim=1) if shared else y_host
        ref = q4.gemv_multi(to_dev_x(x), dm)
        for g, r, (p, s) in zip(got, ref, mats):
            assert torch.equal(g, r.cpu())
            assert rel_inf(g.numpy(), oracle.matmul(x, p, s, threads=8)) <= (2e-3 if x_dtype == "f32" else 1e-2)
    with pytest.raises(ValueError):
        plan.host_step(torch.empty((M, K), dtype=dt), y_host, y_dev=y_dev)        # x not pinned
