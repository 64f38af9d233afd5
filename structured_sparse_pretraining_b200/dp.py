"""Data-parallel plumbing of the layer: one process per GPU.

The weights (and so the static 2:4 mask and its double-pruned copy) are the
same on every rank; each rank runs the whole hot path on its own tokens.
The gradients of the replicated parameters are linear in the tokens, so the
one exchange step is their sum over ranks after the backward pass: the
compressed masked dW and the adapter's dL and dR.  The input gradient dX
stays local, and pruning and double pruning run locally on identical weights.
NCCL carries the sum on GPUs, gloo on the CPU (tests).
"""
import torch
import torch.distributed as dist

WEIGHT_SEED = 0  # every rank draws the same weights and adapter


def token_seed(rank: int) -> int:
    """Seed of a rank's own synthetic tokens (X, dY)."""
    return 1 + rank


def shard(n: int, world: int, rank: int):
    """[start, end) of rank's share of n items split as evenly as possible."""
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def replicated_gradients(dW, dL=None, dR=None):
    """The gradients a data-parallel step sums over ranks, in a fixed order
    (every rank must issue the same collectives in the same order)."""
    return [t for t in (dW, dL, dR) if t is not None]


def allreduce_gradients(tensors, group=None):
    """Sum each tensor over the ranks of `group`, in place, in list order."""
    for t in tensors:
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
