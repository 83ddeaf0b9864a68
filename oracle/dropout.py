"""LoRA dropout on the adapter input (oracle).

Test infrastructure only; see the package docstring.

The adapter branch of the layer reads a dropped-out copy of its input while
the frozen base reads the input itself ("LoRA 与 QLoRA：把大模型微调拆成可负担的
工程", section 4.3, lora_dropout; "QLoRA 量化微调", LoRA dropout in the training
recipe).  Inverted dropout with keep mask D and drop probability p:

    X~ = D (.) X / (1 - p)
    U  = X~ A^T,   Y = X W^T + s U B^T

and, by the chain rule through X~ (dX~/dX = D / (1 - p)), with V = dY B:

    dX = dY W + (D / (1 - p)) (.) (s V A)
    dA = s V^T X~,   dB = s dY^T U

The mask is an input (the random draw), packed one bit per element: bit
(k % 8) of byte [m][k // 8] is D[m][k].  1 - p is taken in fp32, the
precision of the library's scalar argument; the rest is fp64.
"""

import numpy as np

from .linear import lora_scale

F64 = np.float64


def unpack_keep_mask(mask_bytes, K):
    """D (M x K, 0/1 fp64) from the packed bytes (M x K/8 uint8)."""
    b = np.asarray(mask_bytes, dtype=np.uint8)
    bits = (b[:, :, None] >> np.arange(8, dtype=np.uint8)[None, None, :]) & 1
    return bits.reshape(b.shape[0], -1)[:, :K].astype(F64)


def _keep_scale(p):
    return 1.0 / float(np.float32(1.0) - np.float32(p))


def linear_fwd_dropout(w_hat, a, b, alpha, p, mask_bytes, x):
    """Returns (Y, U) in fp64; U = X~ A^T."""
    w, a, b, x = (np.asarray(t, F64) for t in (w_hat, a, b, x))
    d = unpack_keep_mask(mask_bytes, x.shape[1])
    xt = d * x * _keep_scale(p)
    u = xt @ a.T
    y = x @ w.T + lora_scale(alpha, a.shape[0]) * (u @ b.T)
    return y, u


def linear_bwd_dropout(w_hat, a, b, alpha, p, mask_bytes, x, dy):
    """Returns (dX, dA, dB) in fp64."""
    w, a, b, x, dy = (np.asarray(t, F64) for t in (w_hat, a, b, x, dy))
    d = unpack_keep_mask(mask_bytes, x.shape[1])
    k = _keep_scale(p)
    s = lora_scale(alpha, a.shape[0])
    xt = d * x * k
    v = dy @ b
    dx = dy @ w + (d * k) * (s * (v @ a))
    da = s * (v.T @ xt)
    db = s * (dy.T @ (xt @ a.T))
    return dx, da, db
