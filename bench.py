#!/usr/bin/env python3
"""Benchmark of the Q4 (4-bit symmetric, group-32) weight-only GEMV / GEMM on B200.

Headline workload: the LM-head GEMV of a QORA-4B-shaped model -- M=1, K=2560,
N=248,320 (the vocabulary), weights N(0, 0.02^2) with one all-zero group per 1024
rows, bf16 x, f32 y: 358.6 MB of codes, scales, x and y per step, the largest
single-GPU GEMV configuration.  One step = one q4_gemv_multi launch over the head
with the weights declared static (each launch streams its weights while its
predecessor drains).
Metric: effective GB/s = algorithmic bytes (packed codes + binary16 scales + x + f32
y) / device time.  L2 stays cold: the steps alternate between two copies of the head
(717 MB, well above the 126 MB L2).

Timing: the K steps of a run are captured in one CUDA graph; the graph is replayed
at least 10 times and for at least 100 ms, each replay bracketed by CUDA events on
the launching stream (and a barrier under torchrun); the reported time per step is
the median replay divided by K, the maximum over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--rows all|main]

Prints one JSON line (rank 0).  Under torchrun each rank runs its own independent
problem (weak scaling, no collective on the data path).  --impl reference times
the CPU oracle instead (rank 0 only).  Every other configuration (the decode
projections alone and together, the 1024x1024 f32-x GEMV, small batches, the prefill
GEMMs and the extension rows) is reported under "rows", and the oracle is timed on
the host for each configuration under "cpu_baseline.per_config".
"""
from __future__ import annotations

import argparse
import faulthandler
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth_inputs  # noqa: E402

faulthandler.enable()


def log(msg):
    print(f"[bench] {msg}", file=sys.stderr, flush=True)


METRIC = "Q4 GEMV effective GB/s"
UNIT = "GB/s"
MAIN = synth_inputs.LM_HEAD
WORKLOAD = ("LM-head GEMV M=1 K=2560 N=248320 (QORA-4B vocabulary), Q4 group-32 weights N(0,0.02^2) "
            "with one zero group per 1024 rows, bf16 x, f32 y")
MIN_REPLAYS = 10
MIN_TIMED_MS = 100.0
# One config object for both arms (the same workload); each arm's method is reported beside it.
CONFIG = {"workload": WORKLOAD,
          "l2": "every step reads cold weights: the GPU arm alternates two copies of the head (717 MB) "
                "in HBM, above the 126 MB L2; the CPU arm streams its rows from host memory"}


def gemv_bytes(M, N, K, x_bytes=2):
    return N * K // 2 + N * (K // 32) * 2 + M * K * x_bytes + M * N * 4


STEP_BYTES = gemv_bytes(MAIN.M, MAIN.N, MAIN.K)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def kernel_source_hash(name):
    p = os.path.join(ROOT, "bit_weight_only_quantize_b200", "csrc", name)
    return hashlib.sha256(open(p, "rb").read()).hexdigest()[:16]


def recorded_traffic(kernel, workload, src_file):
    """DRAM bytes per launch from the committed ncu summary, if taken on this source."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    want = kernel_source_hash(src_file)
    for line in open(path):
        f = dict(kv.split("=", 1) for kv in line.split() if "=" in kv)
        if f.get("kernel") == kernel and f.get("workload") == workload and f.get("src") == want:
            return float(f["bytes_per_launch"])
    return None


# ---------------------------------------------------------------- clocks (NVML)
REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
           0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
           0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, torch_device):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = "GPU-" + str(torch.cuda.get_device_properties(torch_device).uuid)
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report no clocks rather than guessing
            self.err = str(e)

    def sample(self):
        if not self.ok:
            return
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            self.reasons |= int(self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self.sample()
            time.sleep(0.001)

    def start(self):
        self.samples, self.reasons = [], 0
        self._stop.clear()
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()

    def stop(self):
        self._stop.set()
        self.t.join()

    def report(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "error": getattr(self, "err", "")}
        names = [n for b, n in REASONS.items() if self.reasons & b and b != 0x1]
        med = statistics.median(self.samples) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------- timing helpers
def setup_dist(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(torch, ms, dist, device):
    """The slowest rank's time (every rank gets it); ms itself without a process group."""
    if dist is None:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbs(world, bytes_per_step, steps, ms):
    """Whole-job GB/s: every rank moved bytes_per_step per step, in the slowest rank's time."""
    return world * bytes_per_step * steps / (ms * 1e-3) / 1e9


def replay_count(first_ms, min_replays=MIN_REPLAYS, min_ms=MIN_TIMED_MS):
    """Replays of a graph whose one replay took first_ms: at least min_replays and
    together at least min_ms."""
    return max(min_replays, int(math.ceil(min_ms / max(first_ms, 1e-6))))


def capture(torch, launch, n, stream):
    """One CUDA graph of n launches (launch(i, stream_handle), i = 0 .. n-1)."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            for i in range(n):
                launch(i, stream.cuda_stream)
    return g


def timed_replays(torch, graph, stream, device, dist=None, clocks=None, min_replays=MIN_REPLAYS,
                  min_ms=MIN_TIMED_MS):
    """Replay `graph` (one untimed replay first), each timed replay bracketed by CUDA
    events on `stream`, a device synchronisation and, under torchrun, a barrier; returns
    the list of per-replay milliseconds.  The timed replays follow the warm-up directly,
    so the figure is the burst regime of a kernel timed alone (a load held for longer
    brings in the power cap and lower SM clocks)."""
    with torch.cuda.stream(stream):
        graph.replay()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        graph.replay()
    e1.record(stream)
    torch.cuda.synchronize(device)
    reps = replay_count(e0.elapsed_time(e1), min_replays, min_ms)
    if dist is not None:                              # every rank replays the same number of times
        t = torch.tensor([reps], dtype=torch.int64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        reps = int(t.item())
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    if clocks is not None:
        clocks.start()
    for a, b in ev:
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(device)
        a.record(stream)
        with torch.cuda.stream(stream):
            graph.replay()
        b.record(stream)
        torch.cuda.synchronize(device)
    if clocks is not None:
        clocks.sample()
        clocks.stop()
    if dist is not None:
        dist.barrier()
    return [a.elapsed_time(b) for a, b in ev]


def time_launches(torch, fn, n, device, stream, min_ms=50.0):
    """Median device time of one fn(i) launch: n launches captured in one graph,
    replayed at least 10 times and for at least min_ms; median replay / n."""
    with torch.cuda.stream(stream):
        fn(0)
    torch.cuda.synchronize(device)
    g = capture(torch, lambda i, _s: fn(i), n, stream)
    ms = timed_replays(torch, g, stream, device, min_ms=min_ms)
    del g
    return statistics.median(ms) / n


# ---------------------------------------------------------------- workloads
def bf16_dev(torch, a, device):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def make_quantized(torch, q4, w, seed, device):
    W = synth_inputs.weights(w.weights, w.N, w.K, seed)
    Wd = torch.from_numpy(W).to(device)
    packed, scales = q4.quantize(Wd)
    del Wd
    return W, packed, scales


def rotating_copies(setb, l2, minimum=2):
    """Copies of a working set of setb bytes whose rotation keeps L2 cold (together > 3x L2)."""
    return max(minimum, -(-3 * l2 // max(setb, 1)) + 1)


class LmHeadStep:
    """The LM head, in two copies that alternate, launched through the C ABI."""

    def __init__(self, torch, q4, lib, rank, device):
        import ctypes
        from bit_weight_only_quantize_b200 import _lib as L
        self.lib = lib
        w = MAIN
        self.W, packed, scales = make_quantized(torch, q4, w, rank, device)
        self.copies = 2
        self.pk = [packed, packed.clone()]
        self.sc = [scales, scales.clone()]
        self.rotated_bytes = self.copies * (packed.numel() + scales.numel() * 2)
        self.x_np = synth_inputs.activations(1, w.K, "bf16", rank)
        self.x = bf16_dev(torch, self.x_np, device)
        self.y = torch.empty((1, w.N), dtype=torch.float32, device=device)
        need = q4.gemv_multi_workspace_size(1, w.K, [w.N])
        self.ws = torch.zeros(max(need, 16), dtype=torch.uint8, device=device)
        self._arrays = []
        for c in range(self.copies):
            arr = (L.Weight * 1)()
            arr[0] = L.Weight(self.pk[c].data_ptr(), self.sc[c].data_ptr(), w.N, self.y.data_ptr())
            self._arrays.append((arr, ctypes.cast(arr, ctypes.c_void_p)))
        self.flags = L.WEIGHTS_STATIC

    def launch(self, step, stream_handle):
        st = self.lib.q4_gemv_multi(self.x.data_ptr(), 1, 1, MAIN.K, self._arrays[step % self.copies][1], 1,
                                    self.flags, self.ws.data_ptr(), self.ws.numel(), stream_handle)
        if st != 0:
            raise RuntimeError(f"q4_gemv_multi failed with status {st}")

    def check(self):
        """Max relative error of the last output on sampled rows, against the oracle."""
        import oracle
        rows = np.linspace(0, MAIN.N - 1, 256).astype(np.int64)
        pk = self.pk[0].cpu().numpy().view(np.uint8)
        sc = self.sc[0].cpu().numpy().view(np.uint16)
        ref = oracle.matmul(self.x_np, pk, sc, rows=rows)
        got = self.y.cpu().numpy()[:, rows]
        return float(np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-30))


def measure_main(torch, q4, lib, args, world, rank, device, dist):
    log("setup: quantising the LM head")
    step = LmHeadStep(torch, q4, lib, rank, device)
    stream = torch.cuda.Stream(device=device)
    for i in range(args.warmup):                   # eager warm-up through the same C ABI
        step.launch(i, stream.cuda_stream)
    torch.cuda.synchronize(device)
    log("warm-up done; capturing")
    graph = capture(torch, step.launch, args.steps, stream)
    clocks = ClockSampler(device)
    log(f"clock sampler ok={clocks.ok}; timing")
    reps = timed_replays(torch, graph, stream, device, dist=dist, clocks=clocks)
    ms = statistics.median(reps)
    ms_max = max_over_ranks(torch, ms, dist, device)
    log(f"median replay {ms:.3f} ms over {len(reps)} replays; checking the output")
    err = step.check()
    del graph
    return step, ms_max, reps, clocks.report(), err


def measure_e2e(torch, q4, lib, step, steps, device, dist=None, world=1):
    """Same metric through the C ABI call that takes host buffers (q4_gemv_host): each
    step copies x from pinned host memory, runs the head and copies the f32 logits back
    to pinned host memory before the call returns."""
    n = max(20, min(steps, 2000))
    w = MAIN
    x_host = torch.from_numpy(step.x_np.view(np.int16)).view(torch.bfloat16).pin_memory()
    y_host = torch.empty((1, w.N), dtype=torch.float32).pin_memory()
    x_dev = torch.empty((1, w.K), dtype=torch.bfloat16, device=device)
    stream = torch.cuda.current_stream(device)
    from bit_weight_only_quantize_b200 import _lib as L

    def one(i):
        c = i % step.copies
        st = lib.q4_gemv_host(x_host.data_ptr(), L.Q4_BF16, 1, w.K, step.pk[c].data_ptr(), step.sc[c].data_ptr(),
                              w.N, y_host.data_ptr(), x_dev.data_ptr(), step.y.data_ptr(), L.WEIGHTS_STATIC,
                              step.ws.data_ptr(), step.ws.numel(), stream.cuda_stream)
        if st != 0:
            raise RuntimeError(f"q4_gemv_host failed with status {st}")

    for i in range(3):
        one(i)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    e0.record(stream)
    for i in range(n):
        one(i)
    e1.record(stream)
    torch.cuda.synchronize(device)
    wall = (time.perf_counter() - t0) * 1e3 / n
    ms = max_over_ranks(torch, e0.elapsed_time(e1) / n, dist, device)
    return {"value": job_gbs(world, STEP_BYTES, 1, ms), "unit": UNIT,
            "h2d_bytes_per_step": x_host.numel() * 2,
            "d2h_bytes_per_step": y_host.numel() * 4,
            "steps": n, "ms_per_step": ms, "host_wall_ms_per_step": wall,
            "api": "q4_gemv_host (C ABI): pinned host x -> device, LM-head GEMV, f32 logits -> pinned host, "
                   "stream synchronised in the call"}


def gemv_row(torch, lib, w, packs, x, y, ws, stream, device, hbm, x_bytes=2, name=None):
    """One q4_gemv configuration over rotating weight copies."""
    xt = 0 if x_bytes == 4 else 1

    def fn(i):
        pk, sc = packs[i % len(packs)]
        st = lib.q4_gemv(x.data_ptr(), xt, w.M, w.K, pk.data_ptr(), sc.data_ptr(), w.N, y.data_ptr(),
                         ws.data_ptr(), ws.numel(), stream.cuda_stream)
        assert st == 0
    n = max(len(packs) * 2, 20)
    ms = time_launches(torch, fn, n, device, stream)
    b = gemv_bytes(w.M, w.N, w.K, x_bytes)
    return {"workload": name or f"M={w.M} K={w.K} N={w.N} {'f32' if x_bytes == 4 else 'bf16'} x, q4_gemv",
            "ms": ms, "GB/s": b / ms / 1e6, "frac_hbm": b / ms / 1e6 / hbm, "bytes": b, "launches_per_graph": n,
            "l2": f"{len(packs)} rotating weight copies"}


def measure_rows(torch, q4, lib, device, peaks, l2):
    """Every other configuration and extension row of the library, one GPU."""
    out = {}
    stream = torch.cuda.Stream(device=device)
    hbm = peaks["hbm_gbs"]

    # q4_gemv alone on the small configurations: 1024x1024 with f32 x, and each decode
    # projection shape; rotating copies keep L2 cold.
    for w in [synth_inputs.DECODE_SMALL, *synth_inputs.DECODE_PROJ]:
        _, packed, scales = make_quantized(torch, q4, w, 0, device)
        copies = rotating_copies(packed.numel() + scales.numel() * 2, l2)
        packs = [(packed, scales)] + [(packed.clone(), scales.clone()) for _ in range(copies - 1)]
        xa = synth_inputs.activations(w.M, w.K, w.x_dtype, 0)
        x = torch.from_numpy(xa).to(device) if w.x_dtype == "f32" else bf16_dev(torch, xa, device)
        y = torch.empty((w.M, w.N), dtype=torch.float32, device=device)
        ws = torch.zeros(max(q4.gemv_workspace_size(w.M, w.N, w.K), 16), dtype=torch.uint8, device=device)
        log(f"rows: {w.name}")
        out[w.name] = gemv_row(torch, lib, w, packs, x, y, ws, stream, device, hbm, 4 if w.x_dtype == "f32" else 2)
        del packs

    # The decode step: the three projections of one token in one q4_gemv_multi launch.
    from bit_weight_only_quantize_b200 import _lib as L
    import ctypes
    mats = [make_quantized(torch, q4, w, 0, device) for w in synth_inputs.DECODE_PROJ]
    setb = sum(p.numel() + s.numel() * 2 for _, p, s in mats)
    copies = rotating_copies(setb, l2)
    sets = [[(p, s) for _, p, s in mats]] + [[(p.clone(), s.clone()) for _, p, s in mats] for _ in range(copies - 1)]
    xd = bf16_dev(torch, synth_inputs.activations(1, 2560, "bf16", 0), device)
    ys = [torch.empty((1, w.N), dtype=torch.float32, device=device) for w in synth_inputs.DECODE_PROJ]
    wsd = torch.zeros(max(q4.gemv_multi_workspace_size(1, 2560, [w.N for w in synth_inputs.DECODE_PROJ]), 16),
                      dtype=torch.uint8, device=device)
    arrs = []
    for st_ in sets:
        arr = (L.Weight * 3)()
        for j, ((p, s), w) in enumerate(zip(st_, synth_inputs.DECODE_PROJ)):
            arr[j] = L.Weight(p.data_ptr(), s.data_ptr(), w.N, ys[j].data_ptr())
        arrs.append((arr, ctypes.cast(arr, ctypes.c_void_p)))

    def dec(i):
        st = lib.q4_gemv_multi(xd.data_ptr(), 1, 1, 2560, arrs[i % copies][1], 3, L.WEIGHTS_STATIC, wsd.data_ptr(),
                               wsd.numel(), stream.cuda_stream)
        assert st == 0
    log("rows: decode step")
    n = copies * 2
    ms = time_launches(torch, dec, n, device, stream)
    b = sum(gemv_bytes(1, w.N, w.K) for w in synth_inputs.DECODE_PROJ)
    out["decode_step_3proj"] = {"workload": "decode projections M=1 K=2560 N={2048,4096,1024} bf16 x, one "
                                            "q4_gemv_multi launch, static weights", "ms": ms, "GB/s": b / ms / 1e6,
                                "frac_hbm": b / ms / 1e6 / hbm, "bytes": b, "launches_per_graph": n,
                                "l2": f"{copies} rotating weight sets"}
    del sets, arrs, mats

    # LM head variants (358.6 MB per launch, already far above L2).
    w = synth_inputs.LM_HEAD
    W, packed, scales = make_quantized(torch, q4, w, 0, device)
    x = bf16_dev(torch, synth_inputs.activations(1, w.K, "bf16", 0), device)
    y = torch.empty((1, w.N), dtype=torch.float32, device=device)
    ws = torch.zeros(max(q4.gemv_workspace_size(1, w.N, w.K), 16), dtype=torch.uint8, device=device)
    log("rows: lm head, q4_gemv")
    out["lm_head_q4_gemv"] = gemv_row(torch, lib, w, [(packed, scales)], x, y, ws, stream, device, hbm,
                                      name="M=1 K=2560 N=248320 bf16 x, q4_gemv (no static-weights flag)")

    am_ws = torch.zeros(int(lib.q4_gemv_argmax_workspace_size()), dtype=torch.uint8, device=device)
    am_idx = torch.empty((1,), dtype=torch.int64, device=device)
    am_val = torch.empty((1,), dtype=torch.float32, device=device)

    def lm_argmax(i):
        st = lib.q4_gemv_argmax(x.data_ptr(), 1, 1, w.K, packed.data_ptr(), scales.data_ptr(), w.N, None,
                                am_idx.data_ptr(), am_val.data_ptr(), 1, am_ws.data_ptr(), am_ws.numel(),
                                stream.cuda_stream)
        assert st == 0
    log("rows: lm head argmax")
    ms = time_launches(torch, lm_argmax, 20, device, stream)
    b = w.N * w.K // 2 + w.N * (w.K // 32) * 2 + w.K * 2 + 12
    out["lm_head_argmax"] = {"workload": "greedy step: M=1 K=2560 N=248320 bf16 x, argmax fused, no logits out",
                             "ms": ms, "GB/s": b / ms / 1e6, "frac_hbm": b / ms / 1e6 / hbm, "bytes": b}

    TK = 20
    tk_ws = torch.zeros(max(16, q4.gemv_topk_workspace_size(1, w.N, w.K, TK)), dtype=torch.uint8, device=device)
    tk_idx = torch.empty((1, TK), dtype=torch.int64, device=device)
    tk_val = torch.empty((1, TK), dtype=torch.float32, device=device)

    def lm_topk(i):
        st = lib.q4_gemv_topk(x.data_ptr(), 1, 1, w.K, packed.data_ptr(), scales.data_ptr(), w.N, TK, 0, None,
                              tk_idx.data_ptr(), tk_val.data_ptr(), 1, tk_ws.data_ptr(), tk_ws.numel(),
                              stream.cuda_stream)
        assert st == 0
    log("rows: lm head top-k")
    ms = time_launches(torch, lm_topk, 20, device, stream)
    b = w.N * w.K // 2 + w.N * (w.K // 32) * 2 + w.K * 2 + TK * 12
    out["lm_head_topk20"] = {"workload": "top-k step: M=1 K=2560 N=248320 bf16 x, top-20 fused, no logits out",
                             "ms": ms, "GB/s": b / ms / 1e6, "frac_hbm": b / ms / 1e6 / hbm, "bytes": b,
                             "matches_argmax": bool(torch.equal(tk_idx[:, 0], am_idx)
                                                    and torch.equal(tk_val[:, 0], am_val))}

    # Quantise the LM-head weights: reads 4 B and writes 0.5625 B per weight.
    Wd = torch.from_numpy(W).to(device)
    del W
    pk2 = torch.empty_like(packed)
    sc2 = torch.empty_like(scales)

    def qz(i):
        st = lib.q4_quantize(Wd.data_ptr(), w.N, w.K, pk2.data_ptr(), sc2.data_ptr(), None, stream.cuda_stream)
        assert st == 0
    log("rows: quantize")
    ms = time_launches(torch, qz, 3, device, stream)
    b = w.N * w.K * 4 + w.N * w.K // 2 + w.N * (w.K // 32) * 2
    out["quantize_lm_head"] = {"workload": "W f32 248320x2560 -> Q4", "ms": ms, "GB/s": b / ms / 1e6,
                               "frac_hbm": b / ms / 1e6 / hbm, "bytes": b,
                               "bit_exact_vs_first_encode": bool(torch.equal(pk2, packed) and torch.equal(sc2, scales))}
    del Wd, pk2, sc2, packed, scales

    # Small-batch decode M in {2,4,8,16}, N=4096.
    for sw in synth_inputs.SMALL_BATCH:
        _, packed, scales = make_quantized(torch, q4, sw, 0, device)
        copies = rotating_copies(packed.numel() + scales.numel() * 2, l2)
        packs = [(packed, scales)] + [(packed.clone(), scales.clone()) for _ in range(copies - 1)]
        xs = bf16_dev(torch, synth_inputs.activations(sw.M, sw.K, "bf16", 0), device)
        ysb = torch.empty((sw.M, sw.N), dtype=torch.float32, device=device)
        wss = torch.zeros(max(q4.gemv_workspace_size(sw.M, sw.N, sw.K), 16), dtype=torch.uint8, device=device)
        log(f"rows: gemv m={sw.M}")
        out[sw.name] = gemv_row(torch, lib, sw, packs, xs, ysb, wss, stream, device, hbm)
        del packs

    # Fused MLP gate+up decode (M=1, K=2560, N=4096 per matrix): y = silu(gate) * up.
    gu = synth_inputs.DECODE_PROJ[1]
    _, gpk, gsc = make_quantized(torch, q4, gu, 0, device)
    _, upk, usc = make_quantized(torch, q4, gu, 1, device)
    copies = rotating_copies(2 * (gpk.numel() + gsc.numel() * 2), l2)
    gmats = [(gpk, gsc, upk, usc)] + [(gpk.clone(), gsc.clone(), upk.clone(), usc.clone()) for _ in range(copies - 1)]
    xg = bf16_dev(torch, synth_inputs.activations(1, gu.K, "bf16", 0), device)
    yg = torch.empty((1, gu.N), dtype=torch.float32, device=device)

    def gate_up(i):
        m = gmats[i % copies]
        st = lib.q4_gemv_gate_up(xg.data_ptr(), 1, 1, gu.K, m[0].data_ptr(), m[1].data_ptr(), m[2].data_ptr(),
                                 m[3].data_ptr(), gu.N, yg.data_ptr(), 1, stream.cuda_stream)
        assert st == 0
    log("rows: gate+up")
    ms = time_launches(torch, gate_up, copies * 2, device, stream)
    b = 2 * (gu.N * gu.K // 2 + gu.N * (gu.K // 32) * 2) + gu.K * 2 + gu.N * 4
    out["gate_up_gemv"] = {"workload": "fused gate+up M=1 K=2560 N=4096 x2, bf16 x, y = silu(g)*u", "ms": ms,
                           "GB/s": b / ms / 1e6, "frac_hbm": b / ms / 1e6 / hbm, "bytes": b}
    del gmats

    # F16-weight GEMV (2 bytes per weight), bf16 x.
    for name, N, K in (("f16_gemv_2560x4096", 4096, 2560), ("f16_gemv_lm_head", 248320, 2560)):
        w16 = torch.from_numpy(synth_inputs.weights("normal", N, K, 0).astype(np.float16)).to(device)
        copies = rotating_copies(w16.numel() * 2, l2, minimum=1) if w16.numel() * 2 < 3 * l2 else 1
        ws16 = [w16] + [w16.clone() for _ in range(copies - 1)]
        xf = bf16_dev(torch, synth_inputs.activations(1, K, "bf16", 0), device)
        yf = torch.empty((1, N), dtype=torch.float32, device=device)

        def f16(i, ws16=ws16, xf=xf, yf=yf, N=N, K=K, copies=copies):
            st = lib.q4_f16_gemv(xf.data_ptr(), 1, 1, K, ws16[i % copies].data_ptr(), N, yf.data_ptr(), 1,
                                 stream.cuda_stream)
            assert st == 0
        log(f"rows: {name}")
        ms = time_launches(torch, f16, max(copies * 2, 10), device, stream)
        b = N * K * 2 + K * 2 + N * 4
        out[name] = {"workload": f"F16 weights M=1 K={K} N={N} bf16 x", "ms": ms, "GB/s": b / ms / 1e6,
                     "frac_hbm": b / ms / 1e6 / hbm, "bytes": b}
        del ws16, w16

    # INT8-weight GEMV (the INT8 layers of a mixed INT8/INT4 model).
    N, K = 4096, 2560
    W8 = torch.from_numpy(synth_inputs.weights("outliers", N, K, 0)).to(device)
    codes, sc8 = q4.int8_quantize(W8)
    del W8
    copies = rotating_copies(codes.numel() + sc8.numel() * 2, l2)
    cs = [(codes, sc8)] + [(codes.clone(), sc8.clone()) for _ in range(copies - 1)]
    x8 = bf16_dev(torch, synth_inputs.activations(1, K, "bf16", 0), device)
    y8 = torch.empty((1, N), dtype=torch.float32, device=device)

    def i8(i):
        c, s = cs[i % copies]
        st = lib.q4_int8_gemv(x8.data_ptr(), 1, 1, K, c.data_ptr(), s.data_ptr(), N, y8.data_ptr(),
                              stream.cuda_stream)
        assert st == 0
    log("rows: int8 gemv")
    ms = time_launches(torch, i8, copies * 2, device, stream)
    b = N * K + N * (K // 32) * 2 + K * 2 + N * 4
    out["int8_gemv_2560x4096"] = {"workload": f"INT8 weights M=1 K={K} N={N} bf16 x", "ms": ms, "GB/s": b / ms / 1e6,
                                  "frac_hbm": b / ms / 1e6 / hbm, "bytes": b}
    del cs

    # INT8 weights at the LM-head shape (642 MB, far above L2).
    N = synth_inputs.LM_HEAD.N
    W8 = torch.from_numpy(synth_inputs.weights("normal", N, K, 0)).to(device)
    codes, sc8 = q4.int8_quantize(W8)
    del W8
    yl = torch.empty((1, N), dtype=torch.float32, device=device)

    def i8l(i):
        st = lib.q4_int8_gemv(x8.data_ptr(), 1, 1, K, codes.data_ptr(), sc8.data_ptr(), N, yl.data_ptr(),
                              stream.cuda_stream)
        assert st == 0
    log("rows: int8 gemv lm head")
    ms = time_launches(torch, i8l, 10, device, stream)
    b = N * K + N * (K // 32) * 2 + K * 2 + N * 4
    out["int8_gemv_lm_head"] = {"workload": f"INT8 weights M=1 K={K} N={N} bf16 x", "ms": ms, "GB/s": b / ms / 1e6,
                                "frac_hbm": b / ms / 1e6 / hbm, "bytes": b}
    del codes, sc8, yl

    # A decode layer of mixed precision in one q4_gemv_mixed launch: attention q, k, v in
    # INT8 (4096, 1024, 1024 rows) beside an MLP projection in Q4 (4096 rows), sharing x.
    spec = [(4096, 8), (1024, 8), (1024, 8), (4096, 4)]
    sets = []
    setb = 0
    for i, (n, bits) in enumerate(spec):
        Wm = torch.from_numpy(synth_inputs.weights("outliers", n, K, i)).to(device)
        c, sm = q4.int8_quantize(Wm) if bits == 8 else q4.quantize(Wm)
        sets.append((c, sm, bits))
        setb += c.numel() + sm.numel() * 2
        del Wm
    copies = rotating_copies(setb, l2)
    allsets = [sets] + [[(c.clone(), sm.clone(), bits) for c, sm, bits in sets] for _ in range(copies - 1)]
    ym = [torch.empty((1, n), dtype=torch.float32, device=device) for n, _ in spec]
    wsm = torch.zeros(max(16, q4.gemv_mixed_workspace_size(1, K, spec)), dtype=torch.uint8, device=device)
    arrs = []
    for st_ in allsets:
        arr = (L.MixedWeight * len(spec))()
        for j, ((c, sm, bits), y) in enumerate(zip(st_, ym)):
            arr[j] = L.MixedWeight(c.data_ptr(), sm.data_ptr(), c.shape[0], y.data_ptr(), bits, 0)
        arrs.append((arr, ctypes.cast(arr, ctypes.c_void_p)))

    def mixed(i):
        st = lib.q4_gemv_mixed(x8.data_ptr(), 1, 1, K, arrs[i % copies][1], len(spec), L.WEIGHTS_STATIC,
                               wsm.data_ptr(), wsm.numel(), stream.cuda_stream)
        assert st == 0
    log("rows: mixed int8/q4 layer")
    ms = time_launches(torch, mixed, copies * 2, device, stream)
    b = setb + K * 2 + sum(n for n, _ in spec) * 4
    out["mixed_int8_q4_layer"] = {"workload": "q4_gemv_mixed M=1 K=2560: INT8 q/k/v (4096, 1024, 1024 rows) + Q4 "
                                              "4096 rows, bf16 x, one launch", "ms": ms, "GB/s": b / ms / 1e6,
                                  "frac_hbm": b / ms / 1e6 / hbm, "bytes": b, "l2": f"{copies} rotating weight sets"}
    del allsets, arrs

    # Prefill q4_gemm (bf16 x, bf16 y, f32 accumulate); inputs rotated to exceed 3x L2.
    for gw in synth_inputs.PREFILL:
        _, packed, scales = make_quantized(torch, q4, gw, 0, device)
        xs = bf16_dev(torch, synth_inputs.activations(gw.M, gw.K, "bf16", 0), device)
        copies = rotating_copies(packed.numel() + scales.numel() * 2 + xs.numel() * 2, l2)
        ins = [(xs, packed, scales)] + [(xs.clone(), packed.clone(), scales.clone()) for _ in range(copies - 1)]
        yo = torch.empty((gw.M, gw.N), dtype=torch.bfloat16, device=device)

        def gm(i, ins=ins, yo=yo, gw=gw):
            xx, pp, ss = ins[i % len(ins)]
            st = lib.q4_gemm(xx.data_ptr(), gw.M, gw.K, pp.data_ptr(), ss.data_ptr(), gw.N, yo.data_ptr(),
                             stream.cuda_stream)
            assert st == 0
        log(f"rows: gemm m={gw.M} n={gw.N}")
        n_launch = max(copies, 8)
        ms = time_launches(torch, gm, n_launch, device, stream)
        flops = 2.0 * gw.M * gw.N * gw.K
        tf = flops / ms / 1e9
        out[gw.name] = {"workload": f"M={gw.M} K={gw.K} N={gw.N} bf16 x, bf16 y, q4_gemm", "ms": ms, "TFLOP/s": tf,
                        "frac_bf16_burst": tf / peaks["bf16_tflops"],
                        "frac_bf16_sustained": tf / peaks["bf16_tflops_sustained"],
                        "flops": flops, "l2": f"{copies} rotating input copies"}
        del ins
    torch.cuda.synchronize(device)
    return out


# ---------------------------------------------------------------- CPU oracle baselines
def _oracle_sample(w, seed=0, max_rows=8192, max_x_rows=64):
    """Leading weight rows (and, for a GEMM, leading x rows) of a configuration, quantised
    by the oracle: the bounded sample the host timings run on."""
    import oracle
    n_rows = min(w.N, max_rows)
    W = synth_inputs.weights(w.weights, w.N, w.K, seed, rows=n_rows)
    packed, scales, _ = oracle.quantize(W)
    x = synth_inputs.activations(w.M, w.K, w.x_dtype, seed)
    if w.op == "gemm":
        x = x[:max_x_rows]
    return x, packed, scales


def cpu_oracle_rate(w, sample, threads, budget_s):
    """The oracle as it stands on a bounded sample of one configuration: GB/s for a GEMV
    (packed + scales + x + y of the rows computed), GFLOP/s for a GEMM.  The number of
    weight rows per pass grows from 64 until a pass takes an eighth of the budget; passes
    repeat until the budget is spent."""
    import oracle
    x, packed, scales = sample
    n_all = packed.shape[0]
    r = min(64, n_all)
    while True:
        rows = np.arange(r, dtype=np.int64)
        t0 = time.perf_counter()
        oracle.matmul(x, packed, scales, rows=rows, threads=threads)
        t = time.perf_counter() - t0
        if t >= budget_s / 8 or r == n_all:
            break
        r = min(n_all, r * 4)
    n, t0 = 0, time.perf_counter()
    while True:
        oracle.matmul(x, packed, scales, rows=rows, threads=threads)
        n += 1
        dt = time.perf_counter() - t0
        if dt >= budget_s:
            break
    m = x.shape[0]
    if w.op == "gemv":
        val = gemv_bytes(m, r, w.K, 4 if w.x_dtype == "f32" else 2) * n / dt / 1e9
        unit = "GB/s"
    else:
        val = 2.0 * m * r * w.K * n / dt / 1e9
        unit = "GFLOP/s"
    return {"value": val, "unit": unit, "threads": threads,
            "sample": f"{m} x rows x {r} of {w.N} weight rows, {n} passes in {dt:.2f} s"}


def cpu_baseline(seconds=5.0):
    """The oracle on the host cores: the headline configuration on all cores (a bounded
    sample of the LM head's rows), plus every configuration single-threaded and on all
    cores."""
    import oracle
    cores = min(os.cpu_count() or 1, oracle.max_threads())
    per = {}
    head = None
    for w in [synth_inputs.DECODE_SMALL, *synth_inputs.DECODE_PROJ, synth_inputs.LM_HEAD, *synth_inputs.SMALL_BATCH,
              *synth_inputs.PREFILL]:
        sample = _oracle_sample(w)
        per[w.name] = {"single_thread": cpu_oracle_rate(w, sample, 1, 0.3),
                       "all_cores": cpu_oracle_rate(w, sample, cores, 0.3)}
        if w is MAIN:
            head = cpu_oracle_rate(w, sample, cores, max(1.0, seconds))
    return {"value": head["value"], "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"LM head: {head['sample']} (binary64 oracle, OpenMP over weight rows)",
            "per_config": per}


def run_reference(args, world, rank):
    """The oracle timed on the host as the reference arm (rank 0 only): each step is a
    bounded sample of the LM head's rows, sized so the whole run takes about two minutes."""
    if rank != 0:
        return
    import oracle
    cores = min(os.cpu_count() or 1, oracle.max_threads())
    w = MAIN
    probe_rows = 2048
    W = synth_inputs.weights(w.weights, w.N, w.K, 0, rows=probe_rows)
    packed, scales, _ = oracle.quantize(W)
    x = synth_inputs.activations(1, w.K, "bf16", 0)
    t0 = time.perf_counter()
    oracle.matmul(x, packed, scales, threads=cores)
    t_probe = max(time.perf_counter() - t0, 1e-6)
    budget = 100.0 / max(1, args.steps + args.warmup)
    rows = int(min(w.N, max(probe_rows, probe_rows * budget / t_probe)))
    if rows > probe_rows:
        W = synth_inputs.weights(w.weights, w.N, w.K, 0, rows=rows)
        packed, scales, _ = oracle.quantize(W)
    del W

    def step():
        oracle.matmul(x, packed, scales, threads=cores)
        return gemv_bytes(1, rows, w.K)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    total = 0
    for _ in range(args.steps):
        total += step()
    dt = time.perf_counter() - t0
    value = total / dt / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / max(1, args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": dict(CONFIG, bytes_per_step=STEP_BYTES),
            "method": {"reference": "CPU oracle (scalar C, binary64), no GPU"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"the first {rows} of {w.N} LM-head rows per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- ncu cases
PROFILE_CASES = ["decode", "decode_small", "decode_multi", "lm_head", "lm_head_argmax", "lm_head_topk", "gemv_m2",
                 "gemv_m4", "gemv_m8", "gemv_m16", "gate_up", "f16", "int8", "int8_m4", "int8_quantize", "quantize",
                 "mixed", "gemm", "gemm_m2048", "gemm_m512", "gemm_m512n2048", "topk_merge", "ffma"]


def run_profile_case(args):
    """A few eager launches of one hot-path row, for ncu captures (no timing)."""
    import torch
    import bit_weight_only_quantize_b200 as q4
    from bit_weight_only_quantize_b200 import _lib
    lib = _lib.load()
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device).cuda_stream
    case = args.profile
    n = args.warmup + args.steps

    def x_of(w, seed=0):
        xa = synth_inputs.activations(w.M, w.K, w.x_dtype, seed)
        return torch.from_numpy(xa).to(device) if w.x_dtype == "f32" else bf16_dev(torch, xa, device)

    if case in ("quantize", "int8_quantize"):
        w = synth_inputs.DECODE_PROJ[1]
        Wd = torch.from_numpy(synth_inputs.weights(w.weights, 16 * w.N, w.K, 0)).to(device)   # 168 MB > L2
        for _ in range(n):
            (q4.quantize if case == "quantize" else q4.int8_quantize)(Wd)
    elif case.startswith("gemm"):
        gw = {"gemm": synth_inputs.PREFILL[-2], "gemm_m2048": synth_inputs.PREFILL[2],
              "gemm_m512": synth_inputs.PREFILL[0], "gemm_m512n2048": synth_inputs.PREFILL[1]}[case]
        _, packed, scales = make_quantized(torch, q4, gw, 0, device)
        x = x_of(gw)
        y = torch.empty((gw.M, gw.N), dtype=torch.bfloat16, device=device)
        for _ in range(n):
            assert lib.q4_gemm(x.data_ptr(), gw.M, gw.K, packed.data_ptr(), scales.data_ptr(), gw.N, y.data_ptr(),
                               stream) == 0
    elif case == "decode_multi":
        mats = [make_quantized(torch, q4, w, 0, device) for w in synth_inputs.DECODE_PROJ]
        x = x_of(synth_inputs.DECODE_PROJ[0])
        weights = [(p, s) for _, p, s in mats]
        for _ in range(n):
            q4.gemv_multi(x, weights, weights_static=True)
    elif case in ("lm_head_topk", "lm_head_argmax"):
        w = synth_inputs.LM_HEAD
        _, packed, scales = make_quantized(torch, q4, w, 0, device)
        x = x_of(w)
        for _ in range(n):
            if case == "lm_head_topk":
                q4.gemv_topk(x, packed, scales, 20, weights_static=True)
            else:
                q4.gemv_argmax(x, packed, scales, weights_static=True)
    elif case == "gate_up":
        w = synth_inputs.DECODE_PROJ[1]
        _, gp, gs = make_quantized(torch, q4, w, 0, device)
        _, up, us = make_quantized(torch, q4, w, 1, device)
        x = x_of(w)
        for _ in range(n):
            q4.gemv_gate_up(x, (gp, gs), (up, us))
    elif case == "f16":
        N, K = 248320, 2560
        w16 = torch.from_numpy(synth_inputs.weights("normal", N, K, 0).astype(np.float16)).to(device)
        x = bf16_dev(torch, synth_inputs.activations(1, K, "bf16", 0), device)
        for _ in range(n):
            q4.f16_gemv(x, w16.view(torch.float16))
    elif case in ("int8", "int8_m4"):
        N, K = 4096 * 16, 2560                                            # 168 MB of codes > L2
        W8 = torch.from_numpy(synth_inputs.weights("normal", N, K, 0)).to(device)
        codes, sc8 = q4.int8_quantize(W8)
        del W8
        x = bf16_dev(torch, synth_inputs.activations(1 if case == "int8" else 4, K, "bf16", 0), device)
        for _ in range(n):
            q4.int8_gemv(x, codes, sc8)
    elif case == "mixed":
        K = 2560
        mats = []
        for i, (nr, bits) in enumerate([(4096, 8), (1024, 8), (1024, 8), (4096, 4)]):
            Wm = torch.from_numpy(synth_inputs.weights("outliers", nr, K, i)).to(device)
            c, sm = q4.int8_quantize(Wm) if bits == 8 else q4.quantize(Wm)
            mats.append((c, sm, bits))
        x = bf16_dev(torch, synth_inputs.activations(1, K, "bf16", 0), device)
        for _ in range(n):
            q4.gemv_mixed(x, mats, weights_static=True)
    elif case == "topk_merge":
        S, M, k = 8, 1, 20
        vals = torch.randn((S, M, k), device=device).sort(dim=-1, descending=True).values.contiguous()
        idx = torch.arange(S * M * k, device=device, dtype=torch.int64).view(S, M, k)
        for _ in range(n):
            q4.topk_merge(vals, idx, k)
    else:
        w = {"decode": synth_inputs.DECODE_PROJ[1], "lm_head": synth_inputs.LM_HEAD,
             "decode_small": synth_inputs.DECODE_SMALL, "gemv_m2": synth_inputs.SMALL_BATCH[0],
             "gemv_m4": synth_inputs.SMALL_BATCH[1], "gemv_m8": synth_inputs.SMALL_BATCH[2],
             "gemv_m16": synth_inputs.SMALL_BATCH[3],
             "ffma": synth_inputs.Workload("ffma", "gemv", 2, 2560, 4096, "normal", "f32")}[case]
        _, packed, scales = make_quantized(torch, q4, w, 0, device)
        x = x_of(w)
        y = torch.empty((w.M, w.N), dtype=torch.float32, device=device)
        ws = torch.zeros(max(q4.gemv_workspace_size(w.M, w.N, w.K), 16), dtype=torch.uint8, device=device)
        for _ in range(n):
            assert lib.q4_gemv(x.data_ptr(), 0 if w.x_dtype == "f32" else 1, w.M, w.K, packed.data_ptr(),
                               scales.data_ptr(), w.N, y.data_ptr(), ws.data_ptr(), ws.numel(), stream) == 0
    torch.cuda.synchronize(device)
    print(json.dumps({"profile_case": case, "launches": n}))


# ---------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--rows", choices=["all", "main"], default="all")
    ap.add_argument("--cpu-seconds", type=float, default=5.0)
    ap.add_argument("--profile", choices=["none", *PROFILE_CASES], default="none",
                    help="run a few untimed launches of one row (for ncu) and exit")
    args = ap.parse_args()
    if args.profile != "none":
        run_profile_case(args)
        return
    if args.warmup < 3:
        args.warmup = 3
    args.steps = max(1, args.steps)
    world, rank, local = setup_dist(args)
    if args.impl == "reference":
        run_reference(args, world, rank)
        return

    import torch
    import bit_weight_only_quantize_b200 as q4
    from bit_weight_only_quantize_b200 import _lib

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist_mod
        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
        dist = dist_mod
    lib = _lib.load()
    peaks = load_peaks()

    step, ms, reps, clocks, err = measure_main(torch, q4, lib, args, world, rank, device, dist)
    ms_step = ms / args.steps
    value = job_gbs(world, STEP_BYTES, args.steps, ms)
    per_gpu = STEP_BYTES / (ms_step * 1e-3) / 1e9
    traffic = recorded_traffic("gemv_tma_kernel", "lm_head", "gemv_tma.cu")
    roofline = {"bound": "hbm", "achieved": per_gpu, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": per_gpu / peaks["hbm_gbs"], "traffic": traffic,
                "peak_source": f"{peaks['source']} copy bandwidth (MEASURED_PEAKS.json hbm_gbs), burst: "
                               "the kernel is timed alone",
                "frac_of_8TBps_spec": per_gpu / 8000.0,
                "kernel": "gemv_tma_kernel (M=1 int8 digit-plane path)", "algorithmic_bytes_per_launch": STEP_BYTES,
                "avg_launch_us": ms_step * 1e3}
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": dict(CONFIG, bytes_per_step=STEP_BYTES),
            "method": {"timing": f"graph of {args.steps} steps replayed {len(reps)} times (>= {MIN_REPLAYS} and "
                                 f">= {MIN_TIMED_MS:.0f} ms); CUDA events on the launching stream per replay; "
                                 "median replay / steps; max over ranks",
                       "rotated_bytes": step.rotated_bytes,
                       "replay_ms": {"median": statistics.median(reps), "min": min(reps), "max": max(reps)},
                       "parallelism": f"replicas x{world} (independent problems, no collective)",
                       "check_max_rel_err_sampled_rows": err},
            "roofline": roofline, "gpu_launches": args.steps * len(reps), "clocks": clocks}
    if dist is not None:
        dist.barrier()
    log("e2e")
    line["e2e"] = measure_e2e(torch, q4, lib, step, args.steps, device, dist, world)
    if world == 1:
        del step
        torch.cuda.empty_cache()
        if args.rows == "all":
            props = torch.cuda.get_device_properties(device)
            l2 = int(getattr(props, "L2_cache_size", 126 * 2 ** 20))
            log("other rows")
            line["rows"] = measure_rows(torch, q4, lib, device, peaks, l2)
        log("cpu baseline")
        line["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
