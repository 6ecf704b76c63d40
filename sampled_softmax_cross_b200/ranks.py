"""Per-rank plumbing for data-parallel runs (one process per GPU).

Each rank runs the path on its own microbatch with no collective. Following
``sampled_softmax.py`` (``CandidateBuilder.reset``), rank r of a world of N
starts its negative window at ``V * r // N`` past the common offset, so the
ranks draw different negatives. Timing is the max over ranks.
"""

from __future__ import annotations


def rank_offset(offset: int, V: int, rank: int, world: int) -> int:
    """Window start of `rank`: the common offset staggered by V * rank // world."""
    return (offset + (V * rank) // world) % V


def rank_seed(seed: int, rank: int) -> int:
    """Seed of `rank`'s synthetic microbatch."""
    return seed + rank


def max_over_ranks(value: float, dist, device=None) -> float:
    """Max of a per-rank scalar over the process group (identity without one)."""
    if dist is None or not dist.is_available() or not dist.is_initialized():
        return float(value)
    import torch

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
