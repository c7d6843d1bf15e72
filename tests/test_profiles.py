"""The committed ncu evidence stays consistent with the source: every DRAM-traffic record
names a summary that exists, every ncu command in a summary leaves the GPU clocks alone and
runs only committed files, and the benchmark headline's record was taken on the current
kernel source (otherwise the benchmark line would report no traffic)."""
import os
import re

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PROFILES = os.path.join(ROOT, "profiles")


def _records():
    out = []
    for line in open(os.path.join(PROFILES, "dram_traffic.txt")):
        if line.startswith("#") or not line.strip():
            continue
        out.append(dict(kv.split("=", 1) for kv in line.split()))
    return out


def test_traffic_records_are_complete_and_name_existing_summaries():
    recs = _records()
    assert recs
    for r in recs:
        for key in ("kernel", "workload", "src", "bytes_per_launch", "read", "write", "capture"):
            assert key in r, (key, r)
        assert int(r["bytes_per_launch"]) == int(r["read"]) + int(r["write"])
        assert os.path.exists(os.path.join(ROOT, r["capture"])), r["capture"]


def test_headline_traffic_record_matches_the_current_source():
    assert bench.recorded_traffic("gemv_tma_kernel", "lm_head", "gemv_tma.cu") is not None


def test_ncu_commands_leave_clocks_alone_and_run_committed_files():
    summaries = [f for f in os.listdir(PROFILES) if f.endswith(".md")]
    assert summaries
    for f in summaries:
        text = open(os.path.join(PROFILES, f)).read()
        joined = re.sub(r"\\\n\s*", " ", text)            # shell line continuations
        cmds = re.findall(r"(?m)^\s*(?:\S+=\S+\s+)*ncu\s.*$", joined)
        assert cmds, f"{f} gives no ncu command"
        for c in cmds:
            assert "--clock-control none" in c, (f, c)
        assert "_work" not in text, f
