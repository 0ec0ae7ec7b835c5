"""Multi-process plumbing for replicas of the decode path (one process per GPU).

Decode shards by sequence: sequences are independent, so each rank decodes
its own rows with no data-path exchange.  The only collective is the timing
reduction (max over ranks) after a timed region.
"""
from __future__ import annotations

from typing import List, Sequence

import torch
import torch.distributed as dist


def shard_rows(n_rows: int, rank: int, world: int) -> range:
    """Contiguous, disjoint, covering split of n_rows query rows over world ranks."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    base, extra = divmod(n_rows, world)
    lo = rank * base + min(rank, extra)
    hi = lo + base + (1 if rank < extra else 0)
    return range(lo, hi)


def shard_lengths(seq_lens: Sequence[int], rank: int, world: int) -> List[int]:
    r = shard_rows(len(seq_lens), rank, world)
    return [seq_lens[i] for i in r]


def max_over_ranks(x: float, device=None) -> float:
    """Max of x over the default process group (x itself without one)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
