"""Data-parallel plumbing of the layer: one process per GPU.

The weights (and so the static 2:4 mask and its double-pruned copy) are the
same on every rank; each rank runs the whole hot path on its own tokens.
The gradients of the replicated parameters are linear in the tokens, so the
one exchange step is their sum over ranks after the backward pass: the
compressed masked dW and the adapter's dL and dR.  The input gradient dX
stays local, and pruning and double pruning run locally on identical weights.
NCCL carries the sum on GPUs, gloo on the CPU (tests).

The sum is taken in fp32 whatever the gradients' own format: every gradient
is placed in one flat fp32 bucket (the bf16 dW converted exactly, the fp32 dL
and dR as they are), the bucket is summed over ranks in one collective, and
each gradient is written back, a bf16 one rounded once (nearest even).  A sum
in bf16 would round after every hop of the collective instead.
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


class GradBucket:
    """One fp32 buffer holding every replicated gradient of a step, summed
    over ranks with a single all-reduce.

    `tensors` keep their own storage; fp32 ones may instead be allocated as
    views of the bucket (`view_for`), so that the kernels write them in place
    and only the bf16 gradients are copied in and out."""

    def __init__(self, shapes_dtypes, device):
        self.slots = []
        off = 0
        for shape, dtype in shapes_dtypes:
            n = 1
            for s in shape:
                n *= s
            self.slots.append((off, n, tuple(shape), dtype))
            off += n
        self.flat = torch.zeros(off, dtype=torch.float32, device=device)

    def view_for(self, i):
        """The bucket's fp32 storage of gradient i, shaped like it."""
        off, n, shape, _ = self.slots[i]
        return self.flat[off:off + n].view(shape)

    def allreduce(self, tensors, group=None):
        """Sum `tensors` (in the bucket's order) over the ranks of `group`, in
        place: copy in, one fp32 all-reduce, copy out."""
        assert len(tensors) == len(self.slots)
        for t, (off, n, shape, _) in zip(tensors, self.slots):
            v = self.flat[off:off + n]
            if v.data_ptr() != t.data_ptr():
                v.copy_(t.reshape(-1))
        dist.all_reduce(self.flat, op=dist.ReduceOp.SUM, group=group)
        for t, (off, n, shape, _) in zip(tensors, self.slots):
            v = self.flat[off:off + n]
            if v.data_ptr() != t.data_ptr():
                t.copy_(v.view(shape))


def allreduce_gradients(tensors, group=None):
    """Sum each tensor over the ranks of `group`, in place, in fp32 (one bucket)."""
    b = GradBucket([(t.shape, t.dtype) for t in tensors], tensors[0].device)
    b.allreduce(tensors, group)
