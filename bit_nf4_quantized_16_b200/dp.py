"""Data-parallel plumbing of the QLoRA linear: tokens are sharded over ranks,
the 4-bit weights are replicated, and the only exchange is the sum of the
adapter gradients.

The gradients of the adapters are sums over tokens (dA = s G^T X and
dB = s dY^T H contract over the token index), so the gradient of the whole
batch is the sum over ranks of the gradients of each rank's shard.  This
module holds no compute: torch.distributed does the exchange (NCCL on GPUs,
gloo on CPU), and it imports nothing from the library so that it can be used
and tested without a GPU.
"""

import torch
import torch.distributed as dist


def shard_tokens(m_total: int, rank: int, world: int):
    """[start, end) of this rank's tokens: contiguous, sizes differing by at most one."""
    base, extra = divmod(m_total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def allreduce_adapter_grads(flat_grads: torch.Tensor, group=None):
    """Sum the flattened adapter gradients (all linears, fp32) over the ranks, in place."""
    if dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(flat_grads, op=dist.ReduceOp.SUM, group=group)
    return flat_grads


class OverlappedGradSum:
    """Sums adapter gradients over the ranks while the backward pass goes on.

    The backward pass runs the linears in reverse order; as soon as one
    linear's dA and dB are written, `ready(buf)` starts an asynchronous
    all-reduce of that buffer (a contiguous view of the flattened gradients),
    so the exchange of the last linears' gradients overlaps the backward of
    the earlier ones.  `wait()` blocks the current stream (not the host) on
    every reduction started since the last wait.  Each rank must call
    `ready` on the same buffers in the same order, which holds when every
    rank runs the same layer sequence.  With one rank both calls do nothing.
    """

    def __init__(self, group=None):
        self.group = group
        self.pending = []
        self.active = dist.is_initialized() and dist.get_world_size(group) > 1

    def ready(self, buf: torch.Tensor):
        if self.active:
            self.pending.append(dist.all_reduce(buf, op=dist.ReduceOp.SUM, group=self.group, async_op=True))

    def wait(self):
        for work in self.pending:
            work.wait()
        self.pending = []


def max_over_ranks(value: float, device=None, group=None) -> float:
    """The largest of the ranks' values (a step time measured on each rank)."""
    if not (dist.is_initialized() and dist.get_world_size(group) > 1):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
