"""AdamW for the adapters of one QLoRA linear, one kernel per step.

Only A and B are trained; the 4-bit base stays frozen ("QLoRA技术从入门到精通",
section 3(3)).  The fp32 master copies of A and B, the two AdamW moments and
the gradients share one flat layout - the layout of ``dp.GradBucket`` - so a
step is one ``qlora_adamw`` launch over the whole buffer, which also writes the
bf16 A and B that the linear layer reads.  With ``paged=True`` the moments
sit in managed memory ("LoRA 与 QLoRA：把大模型微调拆成可负担的工程", section
6.3) and can be sent to host memory between steps with ``offload()``.
"""

import torch

from . import qlora as Q
from .dp import GradBucket


class AdapterAdamW:
    """Master weights, moments and bf16 working copies of one adapter pair.

    ``A`` (r x d_in) and ``B`` (d_out x r) are bf16 views for the layer;
    ``master`` holds them in fp32 at the offsets of ``GradBucket``."""

    def __init__(self, A, B, lr, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.0, paged=False):
        r, d_in = A.shape
        d_out = B.shape[0]
        dev = A.device
        lay = GradBucket(r, d_in, d_out, dev)  # the flat layout (its zeros are reused below)
        self.n = lay.flat.numel()
        self.master = lay.flat
        lay.dA.copy_(A.float())
        lay.dB.copy_(B.float())
        self.bf16 = torch.zeros(self.n, dtype=torch.bfloat16, device=dev)
        off_b = lay.off_b
        self.A = self.bf16[:r * d_in].view(r, d_in)
        self.B = self.bf16[off_b:off_b + d_out * r].view(d_out, r)
        self.A.copy_(A)
        self.B.copy_(B)
        self.paged = paged
        if paged:
            self.m = Q.qlora_paged_empty(self.n)
            self.v = Q.qlora_paged_empty(self.n)
        else:
            self.m = torch.zeros(self.n, dtype=torch.float32, device=dev)
            self.v = torch.zeros(self.n, dtype=torch.float32, device=dev)
        self.lr, self.betas, self.eps, self.wd = lr, betas, eps, weight_decay
        self.t = 0
        self.shape = (r, d_in, d_out)

    def grad_bucket(self):
        """A gradient buffer of the same layout for the backward to write into."""
        r, d_in, d_out = self.shape
        return GradBucket(r, d_in, d_out, self.master.device)

    def step(self, bucket, grad_scale=1.0, stream=None):
        """One AdamW step with the gradients in ``bucket`` (already summed over ranks)."""
        assert bucket.flat.numel() == self.n
        if self.paged:
            self.prefetch(True, stream)
        self.t += 1
        Q.qlora_adamw(self.master, bucket.flat, self.m, self.v, self.t, self.lr, self.betas[0],
                      self.betas[1], self.eps, self.wd, grad_scale, param_bf16=self.bf16,
                      stream=stream)

    def prefetch(self, to_device=True, stream=None):
        if self.paged:
            Q.qlora_paged_prefetch(self.m, to_device, stream)
            Q.qlora_paged_prefetch(self.v, to_device, stream)

    def offload(self, stream=None):
        """Send the paged moments to host memory (no-op unless paged)."""
        self.prefetch(False, stream)
