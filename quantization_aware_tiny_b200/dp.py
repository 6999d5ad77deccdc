"""Data-parallel plumbing of the training step (one process per GPU).

The pages' recipe trains with torchrun + DistributedDataParallel: every rank
holds the full (small) weights, quantizes them itself -- the quantizer is
deterministic, so every replica gets identical codes -- runs its own token
shard, and the fp32 weight gradients are summed across ranks.  That sum is
the path's one exchange step; it goes through torch.distributed (NCCL over
NVLink on GPUs, gloo in the CPU tests).
"""
import torch


def shard_seed(base_seed, rank):
    """Seed of a rank's synthetic token shard (weak scaling: distinct tokens,
    the same tokens-per-rank at every world size)."""
    return base_seed + rank


def allreduce_grads(grads, dist_mod):
    """Sum the weight gradients over all ranks, in a fixed order."""
    for g in grads:
        dist_mod.all_reduce(g)


def max_over_ranks(value, dist_mod, device):
    """Largest per-rank value (a timing), the same on every rank."""
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist_mod.all_reduce(t, op=dist_mod.ReduceOp.MAX)
    return float(t.item())
