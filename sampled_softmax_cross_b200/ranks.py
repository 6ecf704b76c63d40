"""Per-rank plumbing for data-parallel runs (one process per GPU).

Each rank runs the path on its own microbatch with no collective inside it.
Following ``sampled_softmax.py`` (``CandidateBuilder.reset``), rank r of a
world of N starts its negative window at ``V * r // N`` past the common
offset, so the ranks draw different negatives. Timing is the max over ranks.

The one exchange of a data-parallel step is the gradient sync of the dense
lm_head gradient: ``allreduce_dw`` sums every rank's ``dW [V, d]`` (bf16)
over the process group, so that every rank holds the sum of the ranks'
gradients -- rows in the union of the ranks' candidate sets carry the sum of
their contributions, all other rows stay exactly +0.0 (each rank's dW is +0.0
off its own C, and a sum of +0.0 terms is +0.0).
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


def allreduce_dw(dW, dist, stream=None):
    """Sum the ranks' dense lm_head gradients in place (NCCL over NVLink on GPUs,
    gloo on CPU tensors). With `stream` (a torch.cuda.Stream) the collective is
    ordered after the work already queued on that stream and the stream waits
    for it; no-op without an initialised process group."""
    if dist is None or not dist.is_available() or not dist.is_initialized():
        return
    if stream is None:
        dist.all_reduce(dW, op=dist.ReduceOp.SUM)
        return
    import torch

    with torch.cuda.stream(stream):
        dist.all_reduce(dW, op=dist.ReduceOp.SUM)
