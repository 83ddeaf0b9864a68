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
"""

import torch
import torch.distributed as dist

_ALIGN = 64  # elements: every view starts on a 256-byte boundary


def token_shard(total_tokens, rank, world):
    """[start, stop) of this rank's tokens when `total_tokens` are split as
    evenly as possible (the first total % world ranks take one more)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside world of size {world}")
    base, extra = divmod(int(total_tokens), world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


class GradBucket:
    """The LoRA gradients of one linear in one flat fp32 buffer.

    ``dA`` (r x K) and ``dB`` (N x r) are contiguous views that the backward
    writes into; ``allreduce`` sums them over the ranks of ``group`` in one
    collective, in place."""

    def __init__(self, r, d_in, d_out, device):
        na = r * d_in
        off_b = -(-na // _ALIGN) * _ALIGN
        self.off_b = off_b
        self.flat = torch.zeros(off_b + d_out * r, dtype=torch.float32, device=device)
        self.dA = self.flat[:na].view(r, d_in)
        self.dB = self.flat[off_b:off_b + d_out * r].view(d_out, r)

    def allreduce(self, group=None, average=False):
        if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
            dist.all_reduce(self.flat, op=dist.ReduceOp.SUM, group=group)
            if average:
                self.flat.div_(dist.get_world_size(group))
        return self


def max_over_ranks(value, device, group=None):
    """The largest of every rank's `value` (a time): a data-parallel step ends
    when its slowest rank does."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
