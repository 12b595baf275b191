"""Multi-GPU plumbing for the one exchange the method has.

Every (batch, head) pair is independent except for dalpha: the LeRoPE log-frequencies
are shared by all heads ("LeRoPE: learnable RoPE frequencies", Escolhas de Design
Principais), so their gradient is the sum over every head of every rank.  Ranks run
their own batches (weak scaling); after each backward the d/2 floats of dalpha are
summed with one all-reduce (NCCL on GPUs, gloo in the CPU tests).
"""
import torch.distributed as dist

RANK_SEED_STRIDE = 7919


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of rank `rank`'s synthetic batch."""
    return base_seed + RANK_SEED_STRIDE * rank


def allreduce_dalpha(dalpha, group=None):
    """In-place sum of every rank's dalpha (shape [d/2], fp32)."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(dalpha, op=dist.ReduceOp.SUM, group=group)
    return dalpha
