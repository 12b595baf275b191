"""Multi-GPU plumbing for the one exchange the method has.

Every (batch, head) pair is independent except for dalpha: the LeRoPE log-frequencies
are shared by all heads ("LeRoPE: learnable RoPE frequencies", Escolhas de Design
Principais), so their gradient is the sum over every head of every rank.  Ranks run
disjoint (batch, head) units -- their own batches (weak scaling, what bench.py times) or
contiguous shards of one batch's B*H units (`shard_bh`) -- and after each backward the
d/2 floats of dalpha are combined by `allreduce_dalpha`: an all-gather of every rank's
partial and a sum in rank order in fp64, so that every rank holds the same bits whatever
the collective's internal reduction order (NCCL on GPUs, gloo in the CPU tests).  The loss
L, a sum over every head as well, is combined the same way.
"""
import torch
import torch.distributed as dist

RANK_SEED_STRIDE = 7919


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of rank `rank`'s synthetic batch."""
    return base_seed + RANK_SEED_STRIDE * rank


def shard_bh(B: int, H: int, world: int, rank: int):
    """(start, count) of rank `rank`'s contiguous share of the B*H (batch, head) units,
    balanced to within one unit.  Rows of a [B, H, n, d] tensor are contiguous per unit,
    so a shard is the [1, count, n, d] problem starting at unit `start`."""
    if not (0 <= rank < world):
        raise ValueError(f"rank {rank} outside world of {world}")
    units = B * H
    base, extra = divmod(units, world)
    start = rank * base + min(rank, extra)
    return start, base + (1 if rank < extra else 0)


def allreduce_sum(x, group=None):
    """x <- the sum of every rank's x (any shape, e.g. dalpha [d/2] or the scalar loss L),
    deterministic: all-gather, then a fixed rank-order fp64 sum on every rank.  A no-op on
    one process."""
    if not (dist.is_available() and dist.is_initialized()):
        return x
    world = dist.get_world_size(group)
    if world == 1:
        return x
    parts = [torch.empty_like(x) for _ in range(world)]
    dist.all_gather(parts, x.contiguous(), group=group)
    acc = torch.zeros(x.shape, dtype=torch.float64, device=x.device)
    for p in parts:  # rank order
        acc += p.to(torch.float64)
    x.copy_(acc.to(x.dtype))
    return x


def allreduce_dalpha(dalpha, group=None):
    """dalpha <- the sum over every rank (see allreduce_sum)."""
    return allreduce_sum(dalpha, group)
