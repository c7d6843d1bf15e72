"""Host logic of the multi-process benchmark on CPU: gloo ranks agree on the slowest
rank's time, the whole-job figure counts every rank's bytes, and the reference arm runs
on rank 0 only and prints a line with the main arm's keys, metric and config."""
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


def test_reference_arm_line_keeps_the_contract(capsys, monkeypatch):
    """On rank 0 the reference arm prints one JSON line with the keys of the main arm's line,
    the same metric, unit and config, and an e2e / cpu_baseline that restate its own value
    (a small head stands in for the LM head so the oracle finishes in well under a second)."""
    import json

    import synth_inputs

    small = synth_inputs.Workload("gemv_2560x4096_small_head", "gemv", 1, 2560, 4096, "lm_head", "bf16")
    monkeypatch.setattr(bench, "MAIN", small)

    class Args:
        steps, warmup, cpu_seconds = 2, 1, 0.01
    bench.run_reference(Args(), 1, 0)
    out = capsys.readouterr().out.strip().splitlines()
    assert len(out) == 1
    line = json.loads(out[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference"
    assert (line["metric"], line["unit"], line["higher_is_better"]) == (bench.METRIC, bench.UNIT, True)
    assert (line["n_gpus"], line["steps"], line["warmup"]) == (1, 2, 1)
    assert line["config"] == dict(bench.CONFIG, bytes_per_step=bench.STEP_BYTES)   # the main arm's config
    assert line["value"] > 0
    # value is the bytes of the sampled rows per step over the time per step
    assert line["value"] * line["ms_per_step"] * 1e6 == pytest.approx(bench.gemv_bytes(1, small.N, small.K))
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["unit"] == line["unit"]
    assert cb["cores"] >= 1 and str(small.N) in cb["sample"]
