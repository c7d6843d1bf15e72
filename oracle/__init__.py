"""Q4 oracle: ctypes wrapper around the scalar C reference in ``q4_oracle.c``.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package.  The product
library never links or calls it, and it imports nothing from the product.

Format and products follow the QORA-4B thread (zingnex.cn, section
"量化与内存管理") and the QORA-LLM-0.8B model card (section "Weight Format"):
4-bit symmetric quantisation, group size 32, one scale per group, products
against the dequantised weights.  The exact encoding is written out in the
header comment of ``q4_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "q4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

FLAG_NONFINITE = 1
FLAG_SCALE_OVERFLOW = 2

_CFLAGS = ["-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared", "-std=c11"]


def build(force: bool = False) -> str:
    """Compile ``q4_oracle.c`` into ``liboracle.so`` next to it (gcc, no SIMD flags)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        i64, vp, i32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
        lib.oracle_f32_to_f16.argtypes = [ctypes.c_float]
        lib.oracle_f32_to_f16.restype = ctypes.c_uint16
        lib.oracle_f16_to_f32.argtypes = [ctypes.c_uint16]
        lib.oracle_f16_to_f32.restype = ctypes.c_float
        lib.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_f32.restype = ctypes.c_float
        lib.oracle_f32_to_f16_array.argtypes = [vp, vp, i64]
        lib.oracle_f32_to_f16_array.restype = None
        lib.oracle_f16_to_f32_array.argtypes = [vp, vp, i64]
        lib.oracle_f16_to_f32_array.restype = None
        lib.oracle_q4_quantize.argtypes = [vp, i64, i64, vp, vp, vp]
        lib.oracle_q4_quantize.restype = i32
        lib.oracle_q4_dequant.argtypes = [vp, vp, i64, i64, vp]
        lib.oracle_q4_dequant.restype = None
        lib.oracle_q4_matmul_rows.argtypes = [vp, i32, i64, i64, vp, vp, vp, i64, vp, i32]
        lib.oracle_q4_matmul_rows.restype = i32
        lib.oracle_q4_matmul.argtypes = [vp, i32, i64, i64, vp, vp, i64, vp, i32]
        lib.oracle_q4_matmul.restype = i32
        lib.oracle_q4_gate_up_rows.argtypes = [vp, i32, i64, i64, vp, vp, vp, vp, vp, i64, vp, i32]
        lib.oracle_q4_gate_up_rows.restype = i32
        lib.oracle_f16_matmul.argtypes = [vp, i32, i64, i64, vp, i64, vp, i32]
        lib.oracle_f16_matmul.restype = i32
        lib.oracle_q8_quantize.argtypes = [vp, i64, i64, vp, vp, vp]
        lib.oracle_q8_quantize.restype = i32
        lib.oracle_q8_matmul.argtypes = [vp, i32, i64, i64, vp, vp, i64, vp, i32]
        lib.oracle_q8_matmul.restype = i32
        lib.oracle_max_threads.argtypes = []
        lib.oracle_max_threads.restype = i32
        _lib = lib
        return lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def f32_to_f16_bits(x) -> np.ndarray:
    """IEEE binary16 round-to-nearest-even of each f32 value, as uint16 bits."""
    a = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(a.shape, dtype=np.uint16)
    _load().oracle_f32_to_f16_array(_ptr(a), _ptr(out), a.size)
    return out


def f16_bits_to_f32(h) -> np.ndarray:
    a = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.empty(a.shape, dtype=np.float32)
    _load().oracle_f16_to_f32_array(_ptr(a), _ptr(out), a.size)
    return out


def quantize(W: np.ndarray):
    """W f32 [N,K] -> (packed uint8 [N,K/2], scales uint16 binary16 bits [N,K/32], flags)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    if K % 32:
        raise ValueError("K must be a multiple of 32")
    packed = np.empty((N, K // 2), dtype=np.uint8)
    scales = np.empty((N, K // 32), dtype=np.uint16)
    flags = np.zeros(1, dtype=np.uint32)
    rc = _load().oracle_q4_quantize(_ptr(W), N, K, _ptr(packed), _ptr(scales), _ptr(flags))
    if rc != 0:
        raise RuntimeError("oracle quantize failed")
    return packed, scales, int(flags[0])


def dequantize(packed: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Exact binary64 dequantised weights [N,K]."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    N, K = packed.shape[0], packed.shape[1] * 2
    out = np.empty((N, K), dtype=np.float64)
    _load().oracle_q4_dequant(_ptr(packed), _ptr(scales), N, K, _ptr(out))
    return out


def matmul(x: np.ndarray, packed: np.ndarray, scales: np.ndarray, rows=None, threads: int = 1) -> np.ndarray:
    """y = x . dequant(W)^T in binary64.

    x: [M,K] float32, or uint16 holding bfloat16 bits.  rows: optional subset of
    output rows (int64 indices); the result then has shape [M, len(rows)].
    """
    if x.dtype == np.uint16:
        is_bf16 = 1
    elif x.dtype == np.float32:
        is_bf16 = 0
    else:
        raise TypeError("x must be float32 or uint16 (bfloat16 bits)")
    x = np.ascontiguousarray(x)
    if x.ndim == 1:
        x = x[None, :]
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    M, K = x.shape
    N = packed.shape[0]
    if packed.shape[1] * 2 != K or scales.shape != (N, K // 32):
        raise ValueError("shape mismatch between x, packed and scales")
    lib = _load()
    if rows is None:
        y = np.empty((M, N), dtype=np.float64)
        rc = lib.oracle_q4_matmul(_ptr(x), is_bf16, M, K, _ptr(packed), _ptr(scales), N, _ptr(y), threads)
    else:
        r = np.ascontiguousarray(rows, dtype=np.int64)
        if r.size and (r.min() < 0 or r.max() >= N):
            raise IndexError("row index out of range")
        y = np.empty((M, r.size), dtype=np.float64)
        rc = lib.oracle_q4_matmul_rows(_ptr(x), is_bf16, M, K, _ptr(packed), _ptr(scales),
                                       _ptr(r), r.size, _ptr(y), threads)
    if rc != 0:
        raise MemoryError("oracle matmul: allocation failed")
    return y


def gate_up(x: np.ndarray, gate, up, rows=None, threads: int = 1) -> np.ndarray:
    """y = silu(x . dequant(Wg)^T) * (x . dequant(Wu)^T) in binary64, silu(g) = g/(1+e^-g).

    The fused gate+up of the QORA-LLM-0.8B model card (section "AVX-512 SIMD
    Acceleration"); the activation is read as SiLU (see ``q4_oracle.c``).
    gate, up: (packed, scales) pairs with equal shapes.  x and rows as for ``matmul``.
    """
    if x.dtype == np.uint16:
        is_bf16 = 1
    elif x.dtype == np.float32:
        is_bf16 = 0
    else:
        raise TypeError("x must be float32 or uint16 (bfloat16 bits)")
    x = np.ascontiguousarray(x)
    if x.ndim == 1:
        x = x[None, :]
    gp, gs = (np.ascontiguousarray(gate[0], dtype=np.uint8), np.ascontiguousarray(gate[1], dtype=np.uint16))
    upk, us = (np.ascontiguousarray(up[0], dtype=np.uint8), np.ascontiguousarray(up[1], dtype=np.uint16))
    M, K = x.shape
    N = gp.shape[0]
    if gp.shape != upk.shape or gs.shape != us.shape or gp.shape[1] * 2 != K or gs.shape != (N, K // 32):
        raise ValueError("shape mismatch between x, gate and up")
    r = np.arange(N, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    if r.size and (r.min() < 0 or r.max() >= N):
        raise IndexError("row index out of range")
    y = np.empty((M, r.size), dtype=np.float64)
    rc = _load().oracle_q4_gate_up_rows(_ptr(x), is_bf16, M, K, _ptr(gp), _ptr(gs), _ptr(upk), _ptr(us), _ptr(r),
                                        r.size, _ptr(y), threads)
    if rc != 0:
        raise MemoryError("oracle gate_up: allocation failed")
    return y


def argmax(x: np.ndarray, packed: np.ndarray, scales: np.ndarray, threads: int = 1):
    """Greedy decoding over an LM head: for each x row, the index and value of the
    largest logit of y = x . dequant(W)^T (binary64), the lowest index on ties.

    The QORA-4B thread (section "量化与内存管理") lists the LM head among the parallel
    workloads; greedy decoding (temperature 0) is the deterministic mode of the
    QORA-LLM-0.8B model card (section "CLI Flags", ``--greedy``).  The index is numpy's
    argmax (first occurrence of the maximum) over the binary64 logits.
    """
    y = matmul(x, packed, scales, threads=threads)
    idx = np.argmax(y, axis=1).astype(np.int64)
    return idx, y[np.arange(y.shape[0]), idx]


def select_topk(values: np.ndarray, indices: np.ndarray, k: int):
    """The k best (value, index) candidates of each row of ``values`` [M, C] (binary64 or
    float32) with row numbers ``indices`` [M, C] (int64): larger value first, the lower
    index among equal values, and a NaN above every number (as numpy's argmax reports a
    NaN).  A candidate with a negative index is padding (the tail of a short list) and
    takes no place.  Returns (index [M, k] int64, value [M, k] float64); when a row has
    fewer than k candidates the tail holds index -1 and value NaN.

    This is the ranking the top-k sampler of the QORA-LLM-0.8B model card (section
    "Sampling Defaults", top_k 20) starts from, written as a plain sort; merging the
    per-shard lists of an N-sharded LM head is the same selection over their union.
    """
    values = np.asarray(values, dtype=np.float64)
    indices = np.asarray(indices, dtype=np.int64)
    if values.shape != indices.shape or values.ndim != 2:
        raise ValueError("values and indices must both be [M, C]")
    if k < 1:
        raise ValueError("k must be at least 1")
    M, C = values.shape
    out_i = np.full((M, k), -1, dtype=np.int64)
    out_v = np.full((M, k), np.nan, dtype=np.float64)
    for m in range(M):
        real = np.nonzero(indices[m] >= 0)[0]
        v, r = values[m, real], indices[m, real]
        nan = np.isnan(v)
        # lexsort sorts by its last key first: NaN first, then larger value, then lower index
        order = np.lexsort((r, -np.where(nan, 0.0, v), ~nan))
        take = order[:k]
        out_i[m, :take.size] = r[take]
        out_v[m, :take.size] = v[take]
    return out_i, out_v


def topk(x: np.ndarray, packed: np.ndarray, scales: np.ndarray, k: int, threads: int = 1, row_base: int = 0):
    """The k largest logits of y = x . dequant(W)^T (binary64) per x row and their rows
    (``row_base`` added, for a shard of a larger LM head), ordered as ``select_topk``."""
    y = matmul(x, packed, scales, threads=threads)
    rows = np.broadcast_to(np.arange(y.shape[1], dtype=np.int64) + row_base, y.shape)
    return select_topk(y, rows, k)


def f16_matmul(x: np.ndarray, w16: np.ndarray, threads: int = 1) -> np.ndarray:
    """y = x . W^T in binary64 for binary16 weights W (the F16 GEMV of the QORA-LLM-0.8B
    model card, section "AVX-512 SIMD Acceleration").  w16: uint16 binary16 bits [N, K];
    x as for ``matmul``."""
    if x.dtype == np.uint16:
        is_bf16 = 1
    elif x.dtype == np.float32:
        is_bf16 = 0
    else:
        raise TypeError("x must be float32 or uint16 (bfloat16 bits)")
    x = np.ascontiguousarray(x)
    if x.ndim == 1:
        x = x[None, :]
    w16 = np.ascontiguousarray(w16, dtype=np.uint16)
    M, K = x.shape
    N = w16.shape[0]
    if w16.ndim != 2 or w16.shape[1] != K:
        raise ValueError("shape mismatch between x and w16")
    y = np.empty((M, N), dtype=np.float64)
    _load().oracle_f16_matmul(_ptr(x), is_bf16, M, K, _ptr(w16), N, _ptr(y), threads)
    return y


def quantize8(W: np.ndarray):
    """INT8 weights, the other half of a mixed INT8/INT4 model (QKV-Core thread, section
    "自适应混合量化"): W f32 [N,K] -> (codes int8 [N,K], scales uint16 binary16 bits
    [N,K/32], flags).  The encoding is written out in ``q4_oracle.c``."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    if W.ndim != 2 or W.shape[1] % 32 != 0:
        raise ValueError("W must be [N, K] with K a multiple of 32")
    N, K = W.shape
    codes = np.empty((N, K), dtype=np.int8)
    scales = np.empty((N, K // 32), dtype=np.uint16)
    flags = ctypes.c_uint32(0)
    if _load().oracle_q8_quantize(_ptr(W), N, K, _ptr(codes), _ptr(scales), ctypes.addressof(flags)) != 0:
        raise ValueError("oracle_q8_quantize rejected the shape")
    return codes, scales, int(flags.value)


def dequantize8(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Exact binary64 INT8 dequantised weights [N,K]: code * f32(scale)."""
    s = f16_bits_to_f32(scales).astype(np.float64)
    return codes.astype(np.float64) * np.repeat(s, 32, axis=1)


def matmul8(x: np.ndarray, codes: np.ndarray, scales: np.ndarray, threads: int = 1) -> np.ndarray:
    """y = x . dequant8(W)^T in binary64; x as for ``matmul``."""
    if x.dtype == np.uint16:
        is_bf16 = 1
    elif x.dtype == np.float32:
        is_bf16 = 0
    else:
        raise TypeError("x must be float32 or uint16 (bfloat16 bits)")
    x = np.ascontiguousarray(x)
    if x.ndim == 1:
        x = x[None, :]
    codes = np.ascontiguousarray(codes, dtype=np.int8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    M, K = x.shape
    N = codes.shape[0]
    if codes.shape != (N, K) or scales.shape != (N, K // 32):
        raise ValueError("shape mismatch between x, codes and scales")
    y = np.empty((M, N), dtype=np.float64)
    _load().oracle_q8_matmul(_ptr(x), is_bf16, M, K, _ptr(codes), _ptr(scales), N, _ptr(y), threads)
    return y


def max_threads() -> int:
    return int(_load().oracle_max_threads())
