"""Host-side helpers for running the forward on several GPUs.

Every (b, h) slab of Longformer attention is independent (the key set N(i)
never crosses samples or heads), so the forward shards without any
collective on the data path: each rank runs lf_attn_fwd on its own slabs.
The only communication is the timing reduction (max over ranks).
"""
from __future__ import annotations

from typing import List, Tuple


def partition_bh(B: int, H: int, world: int) -> List[List[Tuple[int, int, int]]]:
    """Split the B*H slabs over `world` ranks as evenly as possible.

    Returns, per rank, a list of (b, h0, h1) pieces: contiguous head ranges
    of one sample, so each piece is a contiguous [1, h1-h0, T, d] view of a
    [B, H, T, d] tensor that can be passed to lf_attn_fwd as is.
    """
    if B <= 0 or H <= 0 or world <= 0:
        raise ValueError("B, H and world must be positive")
    total = B * H
    out = []
    for rank in range(world):
        lo = total * rank // world
        hi = total * (rank + 1) // world
        pieces = []
        x = lo
        while x < hi:
            b, h0 = divmod(x, H)
            h1 = min(H, h0 + (hi - x))
            pieces.append((b, h0, h1))
            x += h1 - h0
        out.append(pieces)
    return out


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank scalar (a CUDA-event time) over the process group."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(work_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job rate: the work all ranks did over the slowest rank's time."""
    if max_seconds <= 0:
        raise ValueError("time must be positive")
    return work_per_rank * world / max_seconds
