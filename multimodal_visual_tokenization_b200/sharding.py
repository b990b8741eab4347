"""Data-parallel helpers for RVQ tokenization on several GPUs (one process per GPU).

Encode and decode are independent per row, so the multi-GPU path has no data-path
collective: codebooks are replicated and every rank quantizes its own rows.  A packed
batch of native-resolution images is cut only at image boundaries, balanced by token
count (LongCat-2.5 blog, "Supernode-Aware Parallelism" / "Offline Visual Preprocessing":
because image token counts are known when sequences are packed, modality loads can be kept
about even across data-parallel ranks).  Timing uses the max over ranks.
"""
from __future__ import annotations

import bisect


def partition_rows(offsets, world: int) -> list[tuple[int, int]]:
    """Split rows [0, N) into `world` contiguous ranges whose cut points are image
    boundaries (elements of offsets), each cut the boundary nearest the even split
    k*N/world, never moving backwards.  Returns [(start, stop)] per rank."""
    off = [int(v) for v in offsets]
    if world < 1 or not off or off[0] != 0 or any(b < a for a, b in zip(off, off[1:])):
        raise ValueError("offsets must start at 0 and be non-decreasing; world >= 1")
    N = off[-1]
    cuts = [0]
    for k in range(1, world):
        target = k * N / world
        i = bisect.bisect_left(off, target)
        cand = [c for c in (off[i - 1] if i > 0 else None, off[i] if i < len(off) else None) if c is not None]
        best = min(cand, key=lambda c: (abs(c - target), c))
        cuts.append(max(best, cuts[-1]))
    cuts.append(N)
    return [(cuts[r], cuts[r + 1]) for r in range(world)]


def rank_env() -> tuple[int, int, int]:
    import os
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def max_over_ranks(value: float, device=None) -> float:
    """Max of a float over all ranks of the default process group (identity without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())
