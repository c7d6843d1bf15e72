"""Helpers shared by the GPU parity tests: torch <-> numpy plumbing and error measures."""
from __future__ import annotations

import numpy as np
import torch


def to_dev_f32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def to_dev_x(x: np.ndarray) -> torch.Tensor:
    """float32 array, or uint16 bfloat16 bits -> CUDA tensor of the matching dtype."""
    if x.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    return to_dev_f32(x)


def to_np_u8(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint8)


def to_np_u16(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint16)


def rel_inf(y: np.ndarray, ref: np.ndarray) -> float:
    """||y - ref||_inf / ||ref||_inf over the whole output."""
    den = float(np.max(np.abs(ref))) if ref.size else 0.0
    num = float(np.max(np.abs(y.astype(np.float64) - ref))) if ref.size else 0.0
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return num / den


# Unit roundoffs of the two kinds of f32 sums the kernels make.  A CUDA-core f32 add or
# FMA rounds to nearest (u = 2^-24).  An f32 accumulation inside a tensor-core MMA
# instruction (the binary16 GEMV) is not specified to round to nearest; the tests take
# the truncating (round-toward-zero) model for every such sum: u = 2^-23.
U_CUDA_CORE = 2.0 ** -24
U_TENSOR_F32 = 2.0 ** -23


def gamma(n: int, u: float) -> float:
    """gamma_n = n u / (1 - n u): the relative bound of a sum reached through n roundings."""
    return n * u / (1 - n * u)


def x_f64(x: np.ndarray) -> np.ndarray:
    """float32 array, or uint16 bfloat16 bits -> exact float64 values."""
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


def f32_sum_bound(x: np.ndarray, deq: np.ndarray, roundings: int) -> np.ndarray:
    """gamma_n * sum_k |x_k w'_k| per output: the classical bound on an f32 sum of
    exact products reached through at most n round-to-nearest roundings."""
    return gamma(roundings, U_CUDA_CORE) * (np.abs(x_f64(x)) @ np.abs(deq).T)


def mma_path_bound(x: np.ndarray, deq: np.ndarray, roundings: int) -> np.ndarray:
    """Bound for the bf16-activation path of M >= 2: the codes become the bf16 values
    code - 8 exactly, so each product x_k (code_k - 8) is exact in f32; they are summed
    inside the tensor-core MMAs (16 per instruction, chained over the group) and the
    scaled group sums on CUDA cores.  Every rounding is bounded by the tensor-core unit
    roundoff: |y - y_ref| <= gamma_n(2^-23) * sum_k |x_k w'_k|."""
    return gamma(roundings, U_TENSOR_F32) * (np.abs(x_f64(x)) @ np.abs(deq).T)


def digit_shift(x_group: np.ndarray) -> int:
    """The power of two F the M = 1 path scales a box of 256 x values by:
    max |x| * 2^F < 2^30 (F <= 100)."""
    mx = float(np.max(np.abs(x_group))) if x_group.size else 0.0
    if mx == 0.0 or mx < 2.0 ** -126:
        return 100
    e = int(np.floor(np.log2(mx)))
    if 2.0 ** e > mx:              # guard log2 rounding at exact powers of two
        e -= 1
    if 2.0 ** (e + 1) <= mx:
        e += 1
    return min(29 - e, 100)


def digit_path_bound(x: np.ndarray, deq: np.ndarray, roundings: int) -> np.ndarray:
    """Bound for the M = 1 path (K % 256 == 0).  Each box of 256 x values (8 groups) is
    rounded once to integers X = rint(x 2^F) (error <= 2^(-F-1) per element) and cut into
    four base-256 digit planes X_p; the integer MMAs are exact, and plane p's f32 sums
    (CUDA-core FMAs of scale x exact group sums, then 2^-F per box) are bounded by
    gamma_n sum_k |w'_k| |X_p,k| 2^-F.  Scaled by 2^(8 (3 - p)) and summed over p this is
    at most gamma_n sum_k |w'_k| (|x_k| + 1.01 * 2^(24 - F))."""
    xs = x_f64(x)
    wa = np.abs(deq)
    M, K = xs.shape
    out = np.empty((M, deq.shape[0]))
    for m in range(M):
        q = np.repeat(np.array([2.0 ** -digit_shift(xs[m, g:g + 256]) for g in range(0, K, 256)]), 256)[:K]
        out[m] = wa @ (0.5 * q) + gamma(roundings, U_CUDA_CORE) * (wa @ (np.abs(xs[m]) + 1.01 * 2.0 ** 24 * q))
    return out
