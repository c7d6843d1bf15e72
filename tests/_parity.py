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


def f32_sum_bound(x: np.ndarray, deq: np.ndarray, roundings: int) -> np.ndarray:
    """gamma_n * sum_k |x_k w'_k| per output: the classical bound on an f32 sum of
    exact products reached through at most n roundings (u = 2^-24)."""
    u = 2.0 ** -24
    gamma = roundings * u / (1 - roundings * u)
    xa = np.abs(x.astype(np.float64) if x.dtype != np.uint16 else
                (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64))
    return gamma * (xa @ np.abs(deq).T)


def offset_path_bound(x: np.ndarray, scales: np.ndarray, roundings: int) -> np.ndarray:
    """Bound for the bf16-activation decode path, which sums x_k * (128 + code_k) and
    removes 136 * sum(x) per half group: every rounded partial is at most
    144 * s_k * |x_k| per term, so |y - y_ref| <= gamma_n * sum_k |x_k| * 144 * s_k."""
    u = 2.0 ** -24
    gamma = roundings * u / (1 - roundings * u)
    xa = np.abs((x.astype(np.uint32) << 16).view(np.float32).astype(np.float64))
    s = np.repeat(scales.view(np.float16).astype(np.float64), 32, axis=1)
    return gamma * (xa @ (144.0 * s).T)
