"""Data-parallel plumbing for the activation-sparse FFN, one process per GPU.

Inference shards tokens across ranks with no exchange.  A training step has
one exchange: the weight gradients dWg_t, dWu_t, dWd are summed over ranks
(the loss is a sum over all tokens, so each rank's gradients of its own
tokens add up to the full-batch gradients).  The three gradients are views
of one flat fp32 buffer, so a single all-reduce moves them: NCCL over
NVLink / NVSwitch on GPUs, gloo on CPU.  Every rank takes the same
collective calls in the same order.
"""
import torch
import torch.distributed as dist


def shard(T, rank, world):
    """Token range [start, stop) of `rank` among `world` ranks for T tokens:
    contiguous, the first T % world ranks one token longer."""
    if world < 1 or not 0 <= rank < world or T < 0:
        raise ValueError(f"bad shard request T={T} rank={rank} world={world}")
    base, extra = divmod(T, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


class GradBuffer:
    """dWg_t, dWu_t, dWd ([F, d] each) as views of one [3, F, d] buffer."""

    def __init__(self, F, d, device, dtype=torch.float32):
        self.flat = torch.empty((3, F, d), dtype=dtype, device=device)
        self.dWg_t, self.dWu_t, self.dWd = self.flat[0], self.flat[1], self.flat[2]

    def allreduce(self, group=None, async_op=False):
        """Sum the three gradients over the ranks of `group`, in place."""
        return dist.all_reduce(self.flat, op=dist.ReduceOp.SUM, group=group, async_op=async_op)
