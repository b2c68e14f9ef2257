"""Data-parallel decomposition of the EQ-Linear layer over ranks.

Tokens are independent in this layer: the forward pass and the input
gradient of a token depend only on that token, so a batch is split into
contiguous token blocks with no exchange.  The weight and bias gradients are
sums over tokens, so each rank's partial dW/db is summed over ranks (one
all-reduce), the gradient exchange of data-parallel training.
"""
from __future__ import annotations


def shard_range(n_total: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous token block [start, end) of `rank` among `world` ranks
    (sizes differ by at most one)."""
    if world < 1 or not 0 <= rank < world or n_total < 0:
        raise ValueError("bad shard arguments")
    base, extra = divmod(n_total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def allreduce_grads(tensors, group=None):
    """Sum each gradient tensor over the ranks of `group` (in place)."""
    import torch.distributed as dist
    for t in tensors:
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
