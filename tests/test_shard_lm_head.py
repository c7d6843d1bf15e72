"""Host logic of the row-sharded LM head on CPU: the shards cover the rows once, in whole
16-row blocks; over gloo ranks the gathered lists arrive stacked in rank order; and the
top k of the gathered shard lists is the top k of the whole head.  (The per-shard lists
here come from the oracle; on a GPU they come from q4_gemv_topk, tested separately.)"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import synth_inputs
from bit_weight_only_quantize_b200.shard import gather_lists, shard_rows


@pytest.mark.parametrize("N,world", [(248320, 8), (248320, 3), (100, 3), (17, 4), (0, 2), (5, 1)])
def test_shards_cover_rows_once_in_blocks(N, world):
    bounds = [shard_rows(N, world, r) for r in range(world)]
    assert bounds[0][0] == 0 and bounds[-1][1] == N
    for (a0, a1), (b0, _) in zip(bounds, bounds[1:]):
        assert a1 == b0                                  # contiguous, disjoint
    for a0, a1 in bounds:
        assert a0 % 16 == 0 and (a1 % 16 == 0 or a1 == N) and a1 >= a0
    sizes = [(a1 - a0 + 15) // 16 for a0, a1 in bounds]
    assert max(sizes) - min(sizes) <= 1                  # balanced to one block
    with pytest.raises(ValueError):
        shard_rows(N, world, world)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, N, K, k, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        packed, scales, _ = oracle.quantize(synth_inputs.weights("outliers", N, K, seed=3))
        x = synth_inputs.activations(2, K, "bf16", seed=4)
        r0, r1 = shard_rows(N, world, rank)
        idx, val = oracle.topk(x, packed[r0:r1], scales[r0:r1], k, row_base=r0)
        gi, gv = gather_lists(torch.from_numpy(idx), torch.from_numpy(val.astype(np.float32)))
        assert tuple(gi.shape) == (world, 2, k)
        for s in range(world):                          # rank order: list s holds shard s's rows
            s0, s1 = shard_rows(N, world, s)
            live = gi[s][gi[s] >= 0]
            assert bool(((live >= s0) & (live < s1)).all())
        mi, mv = oracle.select_topk(gv.permute(1, 0, 2).reshape(2, -1).numpy(),
                                    gi.permute(1, 0, 2).reshape(2, -1).numpy(), k)
        out[rank] = (mi.tolist(), mv.tolist())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,N,k", [(2, 1000, 20), (3, 70, 32), (4, 40, 20)])
def test_merged_shard_lists_are_the_global_topk(world, N, k):
    K = 256
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank, args=(world, _free_port(), N, K, k, out), nprocs=world, join=True)
    packed, scales, _ = oracle.quantize(synth_inputs.weights("outliers", N, K, seed=3))
    x = synth_inputs.activations(2, K, "bf16", seed=4)
    want_i, want_v = oracle.topk(x, packed, scales, k)
    want_v = want_v.astype(np.float32).astype(np.float64)          # the lists travel as f32
    for r in range(world):
        gi, gv = out[r]
        assert gi == want_i.tolist()                               # every rank, the same global list
        assert np.array_equal(np.array(gv), want_v, equal_nan=True)
