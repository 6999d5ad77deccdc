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


class GradSync:
    """Sums gradients over the ranks while later kernels of the step run.

    start(grads, stream) issues the all-reduce of grads once the work already
    queued on `stream` (the kernels that produced them) is done, without
    making `stream` wait; wait(stream) makes `stream` wait for every started
    all-reduce.  A step calls start for the tied head's gradient as soon as its
    backward is queued, so that sum overlaps the MLP backward, and for the MLP's
    gradients at the end; it waits before the step ends (an optimizer update
    would read the sums).  On CPU tensors (gloo) the calls are plain async
    all-reduces.  Every rank issues the same all-reduces in the same order."""

    def __init__(self, dist_mod):
        self.dist = dist_mod
        self.side = None
        self.works = []

    def start(self, grads, stream=None):
        if grads and grads[0].is_cuda:
            if self.side is None:
                self.side = torch.cuda.Stream(device=grads[0].device)
            main = stream if stream is not None else torch.cuda.current_stream(grads[0].device)
            self.side.wait_stream(main)
            with torch.cuda.stream(self.side):
                for g in grads:
                    self.works.append(self.dist.all_reduce(g, async_op=True))
        else:
            for g in grads:
                self.works.append(self.dist.all_reduce(g, async_op=True))

    def wait(self, stream=None):
        for w in self.works:
            if stream is not None:
                with torch.cuda.stream(stream):
                    w.wait()
            else:
                w.wait()
        if self.side is not None:
            main = stream if stream is not None else torch.cuda.current_stream(self.side.device)
            main.wait_stream(self.side)
        self.works = []


def max_over_ranks(value, dist_mod, device):
    """Largest per-rank value (a timing), the same on every rank."""
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist_mod.all_reduce(t, op=dist_mod.ReduceOp.MAX)
    return float(t.item())
