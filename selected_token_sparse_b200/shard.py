"""Sequence-sharded split-KV across devices: host-side plumbing.

One request's keys are spread over `world` devices, each holding a
contiguous, block-aligned range of every request's positions in its own
paged cache.  Every device runs spa_attention with partial = 1 over its
kv_range (the softmax over its keys, without the sink, and its log-sum-exp);
the partial states are all-gathered and spa_merge_partials combines them,
applying the sink once ("[WebGPU] Add SparsePagedAttention", File summaries:
partial FP32 softmax states merged by a finalize stage).  The arithmetic runs
in libspa's kernels; this module only computes ranges and moves tensors.
"""
from __future__ import annotations

from typing import Optional, Sequence, Tuple

import numpy as np
import torch

from . import spa


def sequence_ranges(lengths: Sequence[int], world: int, rank: int, block_size: int) -> np.ndarray:
    """kv_range [B, 2] int32 of shard `rank` of `world`: request b's positions
    [0, L_b) cut into `world` contiguous pieces at block boundaries (piece r
    starts at block floor(r * nblocks / world)); the last piece runs to L_b."""
    if world < 1 or not 0 <= rank < world or block_size < 1:
        raise ValueError("bad shard geometry")
    out = np.zeros((len(lengths), 2), dtype=np.int32)
    for b, L in enumerate(lengths):
        nblk = (int(L) + block_size - 1) // block_size
        lo = (nblk * rank // world) * block_size
        hi = (nblk * (rank + 1) // world) * block_size if rank + 1 < world else int(L)
        out[b] = (min(lo, int(L)), min(hi, int(L)))
    return out


def shard_block_table(block_table: np.ndarray, ranges: np.ndarray, block_size: int) -> np.ndarray:
    """The block table a shard holds: only the blocks of its own range are
    mapped, every other entry is -1."""
    bt = np.full_like(block_table, -1)
    for b in range(block_table.shape[0]):
        lo, hi = int(ranges[b, 0]), int(ranges[b, 1])
        if hi > lo:
            b0, b1 = lo // block_size, (hi + block_size - 1) // block_size
            bt[b, b0:b1] = block_table[b, b0:b1]
    return bt


def all_gather_partials(part_out: torch.Tensor, part_lse: torch.Tensor,
                        group=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Stack every rank's partial state in rank order: [world, T, H_q, D] and
    [world, T, H_q] (one all-gather each)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    outs = [torch.empty_like(part_out) for _ in range(world)]
    lses = [torch.empty_like(part_lse) for _ in range(world)]
    dist.all_gather(outs, part_out.contiguous(), group=group)
    dist.all_gather(lses, part_lse.contiguous(), group=group)
    return torch.stack(outs), torch.stack(lses)


def merge(part_out: torch.Tensor, part_lse: torch.Tensor, sinks: Optional[torch.Tensor],
          out: torch.Tensor, lse: Optional[torch.Tensor] = None) -> torch.Tensor:
    """spa_merge_partials over gathered partial states."""
    return spa.merge_partials(part_out, part_lse, sinks, out, lse)
