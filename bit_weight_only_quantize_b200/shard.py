"""An LM head split by rows across the ranks of a process group, one GPU per rank.

The QORA-4B thread (section "量化与内存管理") runs the LM head as one of its parallel
workloads; its output rows are independent, so each rank holds whole 16-row blocks of
the Q4 weights and x is replicated.  For greedy decoding (k = 1) or a top-k sampler's
list (QORA-LLM-0.8B model card, section "Sampling Defaults": top_k 20) a rank runs the
fused q4_gemv_topk on its rows, reporting global rows, and the only exchange is an
all-gather of the [M, k] lists (12 bytes per entry per rank); q4_topk_merge then selects
the global top k on every rank.  The logits never leave the ranks' chips.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import gemv_topk, gemv_topk_workspace_size, topk_merge


def shard_rows(N: int, world: int, rank: int) -> tuple[int, int]:
    """Rows [r0, r1) of ``rank``: whole 16-row blocks, spread as evenly as the blocks allow
    (a shard's Q4 rows then start on a 16-byte boundary whenever K % 256 == 0)."""
    if world < 1 or not 0 <= rank < world or N < 0:
        raise ValueError("need world >= 1, 0 <= rank < world and N >= 0")
    blocks = (N + 15) // 16
    return min(N, 16 * (rank * blocks // world)), min(N, 16 * ((rank + 1) * blocks // world))


def gather_lists(index: torch.Tensor, value: torch.Tensor, group=None):
    """Every rank's [M, k] lists, stacked [S, M, k] in rank order (two all-gathers)."""
    world = dist.get_world_size(group)
    M, k = index.shape
    gi = torch.empty((world * M, k), dtype=index.dtype, device=index.device)
    gv = torch.empty((world * M, k), dtype=value.dtype, device=value.device)
    dist.all_gather_into_tensor(gi, index.contiguous(), group=group)
    dist.all_gather_into_tensor(gv, value.contiguous(), group=group)
    return gi.view(world, M, k), gv.view(world, M, k)


class ShardedLMHead:
    """This rank's rows of a Q4 LM head of N rows (``packed``/``scales`` hold rows
    ``shard_rows(N, world, rank)`` of the full encoding)."""

    def __init__(self, packed: torch.Tensor, scales: torch.Tensor, N: int, group=None):
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.N = N
        self.row_base, r1 = shard_rows(N, self.world, rank)
        if packed.shape[0] != r1 - self.row_base or scales.shape[0] != packed.shape[0]:
            raise ValueError(f"this rank holds rows [{self.row_base}, {r1}): got {packed.shape[0]} rows")
        self.packed, self.scales = packed, scales
        self._ws = {}                  # (M, k, x dtype) -> workspace, zero at rest

    def _workspace(self, x: torch.Tensor, k: int) -> torch.Tensor:
        key = (x.shape[0], k, x.dtype)
        if key not in self._ws:
            with torch.cuda.device(x.device):
                size = gemv_topk_workspace_size(x.shape[0], self.packed.shape[0], x.shape[1], k, x.dtype)
            self._ws[key] = torch.zeros(max(16, size), dtype=torch.uint8, device=x.device)
        return self._ws[key]

    def topk(self, x: torch.Tensor, k: int, weights_static: bool = True):
        """(index int64 [M,k], value f32 [M,k]) of the whole head's k largest logits, the
        same on every rank; k = 1 is greedy decoding."""
        idx, val, _ = gemv_topk(x, self.packed, self.scales, k, row_base=self.row_base,
                                workspace=self._workspace(x, k), weights_static=weights_static)
        if self.world == 1:
            return idx, val
        gi, gv = gather_lists(idx, val, self.group)
        return topk_merge(gv, gi, k)
