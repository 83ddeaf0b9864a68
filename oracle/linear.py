"""Forward and backward pass of the QLoRA linear layer (oracle).

Test infrastructure only; see the package docstring.

Forward, "LoRA 与 QLoRA：把大模型微调拆成可负担的工程" section 2:
h = W x + (alpha / r) B A x, with A: r x d_in and B: d_out x r; W frozen.
"QLoRA技术从入门到精通" section 3(2) splits it into the base branch
h_base = W_dequantized x and the LoRA branch h_lora = (B A) x, combined as
h = h_base + (alpha / r) h_lora.  The LoRA branch is evaluated here as
B (A x), equal to (B A) x in exact arithmetic.

Backward, same page section 3(3) and "LoRA 与 QLoRA：把大模型微调拆成可负担
的工程" section 6: W gets no gradient; the gradient reaches A and B and passes
through the dequantised W to the layer input.  For a row-major batch (tokens
as rows) Y = X W^T + s (X A^T) B^T and an upstream gradient dY, calculus gives

    V  = dY B
    dX = dY W + s V A
    dB = s dY^T (X A^T)
    dA = s V^T X

All products are fp64 numpy matmuls of the exactly widened inputs.
"""

import numpy as np

F64 = np.float64


def lora_scale(alpha, r):
    """s = alpha / r, computed once in fp32 (the scalar the kernels use)."""
    return float(np.float32(alpha) / np.float32(r))


def _f64(a):
    return np.asarray(a).astype(F64)


def lora_down(a, x):
    """U = X A^T in fp64: the LoRA branch's first product A x for every token
    row (the pages' A x, with tokens as rows)."""
    return _f64(x) @ _f64(a).T


def linear_fwd(w_hat, a, b, alpha, x):
    """Returns (Y, U) in fp64: U = X A^T, Y = X W^T + s U B^T."""
    w, a, b, x = _f64(w_hat), _f64(a), _f64(b), _f64(x)
    s = lora_scale(alpha, a.shape[0])
    u = lora_down(a, x)
    y = x @ w.T + s * (u @ b.T)
    return y, u


def lora_grads(a, b, alpha, x, dy):
    """Returns (dA, dB) in fp64: the adapters' gradients of the backward pass,
    V = dY B, dB = s dY^T (X A^T), dA = s V^T X.  They need no W; every
    token row contributes a term, so they are taken over all rows given."""
    a, b, x, dy = _f64(a), _f64(b), _f64(x), _f64(dy)
    s = lora_scale(alpha, a.shape[0])
    v = dy @ b
    u = lora_down(a, x)
    return s * (v.T @ x), s * (dy.T @ u)


def linear_bwd(w_hat, a, b, alpha, x, dy):
    """Returns (dX, dA, dB) in fp64; no gradient for W exists."""
    w, a, b, x, dy = _f64(w_hat), _f64(a), _f64(b), _f64(x), _f64(dy)
    s = lora_scale(alpha, a.shape[0])
    v = dy @ b
    dx = dy @ w + s * (v @ a)
    da, db = lora_grads(a, b, alpha, x, dy)
    return dx, da, db


def merge_weight(w_hat, a, b, alpha):
    """W_hat + s B A in fp64: the LoRA update added to the restored weight.

    After training, B A has the shape of W and can be added to it
    ("LoRA 与 QLoRA：把大模型微调拆成可负担的工程" section 3; "LoRA 与 QLoRA：
    用一块 GPU 微调大模型" section LoRA); the 4-bit storage cannot absorb it,
    so the sum goes into a restored 16-bit weight.  The merged bf16 weight is
    this value rounded once to bf16 (``round_to_bf16``), with W_hat the fp32
    dequantised weight.
    """
    w, a, b = _f64(w_hat), _f64(a), _f64(b)
    s = lora_scale(alpha, a.shape[0])
    return w + s * (b @ a)
