"""Seeded synthetic inputs for the QLoRA linear layer.

This module only draws random tensors of the shapes and distributions of the
workloads below; it holds none of the method's arithmetic.  Tests, the
benchmark and the oracle-based checks all take their inputs from here.

Recipe (per linear): W ~ N(0, w_std^2) (d_out x d_in), A ~ N(0, 1/r)
(r x d_in), B ~ N(0, 0.01^2) (d_out x r), X ~ N(0, 1) (M x d_in),
dY ~ N(0, 1) (M x d_out), drawn with torch's CPU generator (or a CUDA
generator when ``device`` is a GPU) seeded with base + 0, 1, 2, 3, 4.
The 7B attention projection adds outliers: a fraction of the entries of W,
chosen uniformly (seed base + 5), set to +-8 w_std with a random sign.
Linear j of layer l in a stack uses base = 16 * (7 l + j).
LoRA A ~ Gaussian, B != 0: the pages' B = 0 initialisation would hide the
LoRA branch, so it is only used as a special case in tests.
"""

import math
from dataclasses import dataclass, field

import torch

LLAMA7B_LINEARS = (  # (name, d_out, d_in) of one decoder layer, 7B shapes
    ("q_proj", 4096, 4096), ("k_proj", 4096, 4096), ("v_proj", 4096, 4096),
    ("o_proj", 4096, 4096), ("gate_proj", 11008, 4096), ("up_proj", 11008, 4096),
    ("down_proj", 4096, 11008),
)
LLAMA65B_LINEARS = (
    ("q_proj", 8192, 8192), ("k_proj", 8192, 8192), ("v_proj", 8192, 8192),
    ("o_proj", 8192, 8192), ("gate_proj", 22016, 8192), ("up_proj", 22016, 8192),
    ("down_proj", 8192, 22016),
)


@dataclass(frozen=True)
class LinearShape:
    d_out: int
    d_in: int
    r: int
    alpha: float
    w_std: float = 0.02
    w_dtype: torch.dtype = torch.bfloat16
    outlier_frac: float = 0.0
    outlier_sigma: float = 8.0


@dataclass(frozen=True)
class Workload:
    name: str
    linears: tuple            # tuple of LinearShape, one per linear of a layer
    tokens: tuple             # token counts M the workload runs at
    layers: int = 1
    notes: str = ""
    extra: dict = field(default_factory=dict)


WORKLOADS = {
    "single_256": Workload(
        "single linear 256x256, r=8", (LinearShape(256, 256, 8, 16.0, w_dtype=torch.float32),), (16,)),
    "attn_4096": Workload(
        "7B attention projection 4096x4096, r=16, 0.1% outliers at 8 sigma",
        (LinearShape(4096, 4096, 16, 32.0, outlier_frac=0.001),), (4096,)),
    "mlp_11008": Workload(
        "7B MLP gate/up 4096->11008 and down 11008->4096, r=64",
        (LinearShape(11008, 4096, 64, 16.0), LinearShape(4096, 11008, 64, 16.0)), (1, 16, 8192)),
    "stack_7b": Workload(
        "7B decoder stack, 32 layers x 7 linears, r=16",
        tuple(LinearShape(o, i, 16, 32.0) for _, o, i in LLAMA7B_LINEARS), (2048,), layers=32),
    "stack_65b": Workload(
        "65B linears, 80 layers x 7 linears, r=64",
        tuple(LinearShape(o, i, 64, 16.0, w_std=0.015) for _, o, i in LLAMA65B_LINEARS), (2048,), layers=80),
}


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def randn(shape, std, seed, dtype, device="cpu"):
    """N(0, std^2) drawn in fp32 from a seeded generator, then cast."""
    t = torch.randn(shape, generator=_gen(seed, device), device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def weight(shape: LinearShape, base_seed=0, device="cpu"):
    w = randn((shape.d_out, shape.d_in), shape.w_std, base_seed + 0, torch.float32, device)
    if shape.outlier_frac > 0:
        n = w.numel()
        k = max(1, int(round(shape.outlier_frac * n)))
        g = _gen(base_seed + 5, device)
        pos = torch.randperm(n, generator=g, device=device)[:k]
        sign = torch.randint(0, 2, (k,), generator=g, device=device).to(torch.float32) * 2 - 1
        w.view(-1)[pos] = sign * shape.outlier_sigma * shape.w_std
    return w.to(shape.w_dtype)


def lora_a(shape: LinearShape, base_seed=0, device="cpu"):
    return randn((shape.r, shape.d_in), 1.0 / math.sqrt(shape.r), base_seed + 1, torch.bfloat16, device)


def lora_b(shape: LinearShape, base_seed=0, device="cpu"):
    return randn((shape.d_out, shape.r), 0.01, base_seed + 2, torch.bfloat16, device)


def activations(shape: LinearShape, m, base_seed=0, device="cpu"):
    return randn((m, shape.d_in), 1.0, base_seed + 3, torch.bfloat16, device)


def grad_output(shape: LinearShape, m, base_seed=0, device="cpu"):
    return randn((m, shape.d_out), 1.0, base_seed + 4, torch.bfloat16, device)


def linear_inputs(shape: LinearShape, m, base_seed=0, device="cpu"):
    """All inputs of one linear: W, A, B, X, dY."""
    return dict(W=weight(shape, base_seed, device), A=lora_a(shape, base_seed, device),
                B=lora_b(shape, base_seed, device), X=activations(shape, m, base_seed, device),
                dY=grad_output(shape, m, base_seed, device))


def stack_seed(layer, j):
    return 16 * (7 * layer + j)
