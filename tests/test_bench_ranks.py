"""Host logic of the multi-process benchmark on CPU: gloo ranks agree on the slowest
rank's time, the whole-job figure counts every rank's bytes, and the reference arm runs
on rank 0 only."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out[rank] = bench.max_over_ranks(torch, times[rank], dist, torch.device("cpu"))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ranks_agree_on_the_slowest_time(world):
    times = [1.5, 4.25, 2.0][:world]
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank, args=(world, _free_port(), times, out), nprocs=world, join=True)
    assert [out[r] for r in range(world)] == [max(times)] * world


def test_no_process_group_keeps_the_local_time():
    assert bench.max_over_ranks(torch, 3.0, None, torch.device("cpu")) == 3.0


def test_job_value_counts_every_rank():
    one = bench.job_gbs(1, bench.STEP_BYTES, 100, 2.0)
    assert bench.job_gbs(4, bench.STEP_BYTES, 100, 2.0) == pytest.approx(4 * one)
    assert one == pytest.approx(bench.STEP_BYTES * 100 / 2e-3 / 1e9)


def test_reference_arm_prints_on_rank_zero_only(capsys, monkeypatch):
    class Args:
        steps, warmup, cpu_seconds = 1, 0, 0.01
    monkeypatch.setattr(bench, "cpu_baseline", lambda *a, **k: {"value": 1.0})
    bench.run_reference(Args(), 2, 1)
    assert capsys.readouterr().out == ""
