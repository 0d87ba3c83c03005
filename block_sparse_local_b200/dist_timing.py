"""Multi-rank plumbing of bench.py: independent problems per rank and the
max-over-ranks reduction of device timings.

STA shards into independent (batch, head) problems, so ranks exchange no
data: each rank draws its own batch element from a rank-specific seed, and
the only collective is the reduction of the timed milliseconds (the job is as
slow as its slowest rank).
"""
import torch
import torch.distributed as dist


def rank_seed(base, rank):
    """Seed of rank ``rank``'s batch element (distinct per rank)."""
    return base + 17 * rank


def max_over_ranks(values, device=None):
    """Element-wise max of ``values`` (floats) over all ranks of the default
    process group; identity when it is not initialised or has one rank."""
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]
