"""Several LoRA adapters over one quantised base (oracle).

Test infrastructure only; see the package docstring.

"LoRA 与 QLoRA：把大模型微调拆成可负担的工程" section 3: the base weights are
shared and each task keeps only its own small pair (A, B), picked per
request.  Here n adapters of rank r share W; token m uses adapter
ids[m] (no adapter when the id is outside [0, n)).  For the tokens of
adapter a (rows R_a) the layer and its gradients are the single-adapter ones
restricted to those rows:

    Y[R_a]  = X[R_a] W^T + s (X[R_a] A_a^T) B_a^T
    dX[R_a] = dY[R_a] W + s (dY[R_a] B_a) A_a
    dA_a    = s (dY[R_a] B_a)^T X[R_a]
    dB_a    = s dY[R_a]^T (X[R_a] A_a^T)

and tokens without an adapter see the base layer only.  The adapters are
given as lists; results for A and B come back stacked along the rank
(dA: (n r) x d_in, dB: d_out x (n r)), and U as M x (n r) with each token's
X A_a^T in its own adapter's columns and zeros elsewhere.  fp64 throughout.
"""

import numpy as np

from .linear import lora_scale

F64 = np.float64


def _rows(ids, a):
    return np.nonzero(np.asarray(ids) == a)[0]


def linear_fwd_multi(w_hat, a_list, b_list, alpha, x, ids):
    """Returns (Y, U) in fp64."""
    w, x = np.asarray(w_hat, F64), np.asarray(x, F64)
    n, r = len(a_list), np.asarray(a_list[0]).shape[0]
    s = lora_scale(alpha, r)
    y = x @ w.T
    u = np.zeros((x.shape[0], n * r), F64)
    for a in range(n):
        rows = _rows(ids, a)
        if rows.size == 0:
            continue
        ua = x[rows] @ np.asarray(a_list[a], F64).T
        u[rows, a * r:(a + 1) * r] = ua
        y[rows] += s * (ua @ np.asarray(b_list[a], F64).T)
    return y, u


def linear_bwd_multi(w_hat, a_list, b_list, alpha, x, dy, ids):
    """Returns (dX, dA stacked, dB stacked) in fp64."""
    w, x, dy = np.asarray(w_hat, F64), np.asarray(x, F64), np.asarray(dy, F64)
    n, r = len(a_list), np.asarray(a_list[0]).shape[0]
    s = lora_scale(alpha, r)
    dx = dy @ w
    da = np.zeros((n * r, x.shape[1]), F64)
    db = np.zeros((w.shape[0], n * r), F64)
    for a in range(n):
        rows = _rows(ids, a)
        if rows.size == 0:
            continue
        aa, bb = np.asarray(a_list[a], F64), np.asarray(b_list[a], F64)
        v = dy[rows] @ bb
        dx[rows] += s * (v @ aa)
        da[a * r:(a + 1) * r] = s * (v.T @ x[rows])
        db[:, a * r:(a + 1) * r] = s * (dy[rows].T @ (x[rows] @ aa.T))
    return dx, da, db
