"""Seeded synthetic inputs for the Q4 weight-only GEMV / GEMM workloads.

This module only draws random numbers and shapes them; it holds none of the
quantiser's or the products' arithmetic.  Both the CUDA library's tests and the
oracle consume the arrays it returns.

Recipes (seeded numpy ``default_rng``; weights from stream ``[seed, 0]``, x from
``[seed, 1]``, outlier / zero-group positions from ``[seed, 2]``):

* ``normal``: W ~ N(0, 0.02^2) f32.
* ``outliers``: ``normal`` plus, in exactly round(0.01 * N*K/32) groups drawn
  without replacement, one uniformly chosen element multiplied by 8.
* ``lm_head``: ``normal``, and for every row r with r % 1024 == 0 the group
  (r // 1024) % (K/32) set to 0.0.
* ``student_t``: W = 0.02 * Student-t(nu=4) f32.
* x ~ N(0, 1) f32; a bfloat16 x is the round-to-nearest-even cast of that f32
  array (torch's CPU cast), handed over as uint16 bit patterns.

The shapes follow the QORA-4B thread (zingnex.cn, section "模型规格": hidden
2560, vocabulary 248,320; DeltaNet 16 QK / 32 V heads of 128, full attention
16 Q / 4 KV heads of 256), which give K=2560 and N in {1024, 2048, 4096, 248320}.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

WEIGHT_STD = 0.02


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.default_rng([seed, stream])


def weights(kind: str, N: int, K: int, seed: int = 0, rows: int | None = None) -> np.ndarray:
    """f32 [N,K] weight matrix drawn by recipe ``kind``; with ``rows``, only its first
    ``rows`` rows (the same values, drawn without the rest of the matrix)."""
    if K % 32:
        raise ValueError("K must be a multiple of 32")
    n = N if rows is None else max(0, min(rows, N))
    if kind == "outliers" and n < N:
        return weights(kind, N, K, seed)[:n]       # outlier positions are drawn over the whole matrix
    r = _rng(seed, 0)
    if kind == "student_t":
        W = (WEIGHT_STD * r.standard_t(4.0, size=(n, K))).astype(np.float32)
    else:
        W = r.normal(0.0, WEIGHT_STD, size=(n, K)).astype(np.float32)
    if kind in ("normal", "student_t"):
        return W
    pos = _rng(seed, 2)
    G = K // 32
    if kind == "outliers":
        n_out = int(round(0.01 * N * G))
        if n_out:
            flat = pos.choice(N * G, size=n_out, replace=False)
            rows, groups = np.divmod(flat, G)
            elem = pos.integers(0, 32, size=n_out)
            W[rows, groups * 32 + elem] *= np.float32(8.0)
        return W
    if kind == "lm_head":
        for r0 in range(0, n, 1024):
            g = (r0 // 1024) % G
            W[r0, g * 32:(g + 1) * 32] = 0.0
        return W
    raise ValueError(f"unknown weight recipe {kind!r}")


def activations_f32(M: int, K: int, seed: int = 0) -> np.ndarray:
    return _rng(seed, 1).normal(0.0, 1.0, size=(M, K)).astype(np.float32)


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even bfloat16 cast (torch CPU), returned as uint16 bits."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def activations(M: int, K: int, dtype: str, seed: int = 0) -> np.ndarray:
    """x [M,K]: float32 array, or uint16 bfloat16 bits when dtype == 'bf16'."""
    x = activations_f32(M, K, seed)
    if dtype == "f32":
        return x
    if dtype == "bf16":
        return to_bf16_bits(x)
    raise ValueError(dtype)


@dataclass(frozen=True)
class Workload:
    """One product shape of the benchmark configurations."""
    name: str
    op: str          # "gemv" or "gemm"
    M: int
    K: int
    N: int
    weights: str     # recipe for weights()
    x_dtype: str     # "f32" or "bf16"


# The configurations the benchmark and the parity tests use.
DECODE_SMALL = Workload("gemv_1024x1024_f32x", "gemv", 1, 1024, 1024, "normal", "f32")
DECODE_PROJ = [
    Workload(f"gemv_2560x{n}_proj", "gemv", 1, 2560, n, "outliers", "bf16") for n in (2048, 4096, 1024)
]
LM_HEAD = Workload("gemv_2560x248320_lmhead", "gemv", 1, 2560, 248320, "lm_head", "bf16")
SMALL_BATCH = [Workload(f"gemv_m{m}_2560x4096", "gemv", m, 2560, 4096, "student_t", "bf16") for m in (2, 4, 8, 16)]
PREFILL = [
    Workload(f"gemm_m{m}_2560x{n}", "gemm", m, 2560, n, "normal", "bf16")
    for m in (512, 2048, 8192) for n in (4096, 2048)
]
ALL = [DECODE_SMALL, *DECODE_PROJ, LM_HEAD, *SMALL_BATCH, *PREFILL]


def make(w: Workload, seed: int = 0):
    """(W f32 [N,K], x [M,K]) for workload ``w``."""
    return weights(w.weights, w.N, w.K, seed), activations(w.M, w.K, w.x_dtype, seed)
