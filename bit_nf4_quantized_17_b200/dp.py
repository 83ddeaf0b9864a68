"""Data-parallel replicas of the QLoRA linear layer.

The frozen NF4 base weight receives no gradient: only the adapters A and B are
updated ("QLoRA技术从入门到精通", section 3, QLoRA工作流程; "LoRA 与 QLoRA：把
大模型微调拆成可负担的工程", section 6).  Data parallelism therefore needs no exchange in
the forward pass or for dX: every rank holds the same quantised W and the same
A, B and runs its own tokens.  The LoRA gradients are sums over tokens,

    dA = s V^T X = s sum_ranks V_rank^T X_rank,
    dB = s dY^T U = s sum_ranks dY_rank^T U_rank,

so one all-reduce (sum) of dA and dB per step gives every rank the gradient
of the whole batch.  dA and dB live as views in one flat fp32 buffer so that
the exchange is a single collective (NCCL over NVLink on GPUs, gloo on CPU).
A stack of layers keeps one such buffer per layer (``LayerBucket``): the
exchange of a layer's buffer is started as soon as its backward is enqueued
and runs beside the backward of the layer below.
"""

import torch
import torch.distributed as dist

_ALIGN = 64  # elements: every view starts on a 256-byte boundary


def _aligned(n):
    return -(-int(n) // _ALIGN) * _ALIGN


def token_shard(total_tokens, rank, world):
    """[start, stop) of this rank's tokens when `total_tokens` are split as
    evenly as possible (the first total % world ranks take one more)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside world of size {world}")
    base, extra = divmod(int(total_tokens), world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def _world(group):
    if dist.is_available() and dist.is_initialized():
        return dist.get_world_size(group)
    return 1


class LayerBucket:
    """The LoRA gradients of several linears in one flat fp32 buffer.

    ``shapes`` lists (r, d_in, d_out) per linear; ``views[j]`` is the pair
    (dA_j r x d_in, dB_j d_out x r) of contiguous views, each starting on a
    256-byte boundary, in the order given.  ``allreduce`` sums the whole
    buffer over the ranks of ``group`` in one collective, in place; with
    ``async_op`` it returns the collective's work handle (None on one rank),
    which the caller waits on before reading the sums."""

    def __init__(self, shapes, device):
        spans = []
        off = 0
        for r, d_in, d_out in shapes:
            a = off
            off = _aligned(a + r * d_in)
            b = off
            off = _aligned(b + d_out * r)
            spans.append((a, b, r, d_in, d_out))
        self.flat = torch.zeros(max(off, 1), dtype=torch.float32, device=device)
        self.spans = spans
        self.views = [(self.flat[a:a + r * k].view(r, k), self.flat[b:b + n * r].view(n, r))
                      for a, b, r, k, n in spans]

    def allreduce(self, group=None, average=False, async_op=False):
        if _world(group) == 1:
            return None if async_op else self
        work = dist.all_reduce(self.flat, op=dist.ReduceOp.SUM, group=group, async_op=async_op)
        if average:
            if async_op:
                raise ValueError("average with async_op: divide after waiting")
            self.flat.div_(_world(group))
        return work if async_op else self


class GradBucket(LayerBucket):
    """The LoRA gradients of one linear: ``dA`` (r x K) and ``dB`` (N x r) are
    views of ``flat`` at offsets 0 and ``off_b``."""

    def __init__(self, r, d_in, d_out, device):
        super().__init__([(r, d_in, d_out)], device)
        self.off_b = self.spans[0][1]
        self.dA, self.dB = self.views[0]


def max_over_ranks(value, device, group=None):
    """The largest of every rank's `value` (a time): a data-parallel step ends
    when its slowest rank does."""
    if _world(group) == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
