"""Host-side logic for running the path on several GPUs, one process per GPU.

The scan has no exchange step: sequences (and value heads) are independent, so a batch is
split across ranks and each rank runs the whole path on its share; nothing crosses
NVLink on the data path. Timing is the maximum over ranks.
"""
from __future__ import annotations

import numpy as np


def balance_sequences(seqlens, world: int):
    """Assign sequences to `world` ranks so that token counts are balanced: longest first,
    each to the currently lightest rank. Returns a list of index lists (sorted)."""
    order = sorted(range(len(seqlens)), key=lambda i: (-int(seqlens[i]), i))
    loads = [0] * world
    parts = [[] for _ in range(world)]
    for i in order:
        r = min(range(world), key=lambda j: (loads[j], j))
        parts[r].append(i)
        loads[r] += int(seqlens[i])
    return [sorted(p) for p in parts]


def shard_range(n: int, world: int, rank: int):
    """Contiguous [begin, end) share of n units for `rank`."""
    return n * rank // world, n * (rank + 1) // world


def pack(seqlens, index):
    """cu_seqlens of the sub-batch made of sequences `index` and, for each, its token slice
    in the full packed batch."""
    full = np.zeros(len(seqlens) + 1, dtype=np.int64)
    full[1:] = np.cumsum(np.asarray(seqlens, dtype=np.int64))
    cu = np.zeros(len(index) + 1, dtype=np.int32)
    cu[1:] = np.cumsum([int(seqlens[i]) for i in index])
    slices = [slice(int(full[i]), int(full[i + 1])) for i in index]
    return cu, slices


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank scalar over the default process group (identity without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
