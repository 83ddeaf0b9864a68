"""GPU parity of the linear layer for the pages' quantisation variants.

Block sizes other than 64, double quantisation off (fp32 absmax per block,
4.5 bit/weight) and the uniform 16-level grid ("QLoRA技术从入门到精通", 2(3)
存索引号查找映射表: uniform grid and NF4 grid; "QLoRA 量化微调", 7.1 for the
4.5-bit storage; "大模型瘦身术", 4.1 for block sizes 64 / 256 / 1024), on every
path of the library: the CTA-pair kernels (many tokens), the split-K
single-CTA kernel, the decode forward with W in tensor memory, the dX GEMV
(one token) and the CUDA-core fallback (r not a multiple of 8).  Codes are
compared bit for bit, forward and backward within the stated tolerance.
"""

import numpy as np
import pytest
import torch

import oracle
from bit_nf4_quantized_17_b200 import qlora as Q
from bit_nf4_quantized_17_b200 import workloads as WL
from parity import assert_close, assert_close_scaled, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"

VARIANTS = [  # blocksize, dq_blocksize, table
    (128, 256, Q.QLORA_TABLE_NF4),
    (256, 0, Q.QLORA_TABLE_NF4),
    (1024, 256, Q.QLORA_TABLE_UNIFORM),
    (64, 0, Q.QLORA_TABLE_UNIFORM),
    (512, 64, Q.QLORA_TABLE_NF4),
]

SHAPES = [  # M, N, K, r: which path
    (4096, 2560, 1024, 16),  # CTA pairs
    (700, 384, 2048, 16),    # single-CTA kernel, split contraction
    (3, 256, 1024, 16),      # decode forward (W in TMEM), tensor-core dX
    (1, 264, 1024, 8),       # decode forward, dX GEMV
    (5, 96, 2048, 5),        # CUDA-core fallback
]


def _levels(table):
    return oracle.uniform_levels() if table == Q.QLORA_TABLE_UNIFORM else oracle.nf4_levels()


@pytest.mark.parametrize("bs,dq,table", VARIANTS,
                         ids=[f"b{b}-dq{d}-{'uni' if t else 'nf4'}" for b, d, t in VARIANTS])
@pytest.mark.parametrize("M,N,K,r", SHAPES, ids=["pairs", "splitk", "decode", "gemv", "simt"])
def test_linear_variants(bs, dq, table, M, N, K, r):
    shape = WL.LinearShape(N, K, r, 2.0 * r)
    inp = WL.linear_inputs(shape, M, 31 * bs + K + M)
    inp["B"] = WL.randn((N, r), 0.05, 77 + r, torch.bfloat16)
    W, A, B, X, dY = (inp[k] for k in ("W", "A", "B", "X", "dY"))
    q = Q.qlora_quantize(W.to(DEV), blocksize=bs, dq_blocksize=dq, table=table)
    ref = oracle.quantize(W.float().numpy(), bs, dq, levels=_levels(table))
    assert np.array_equal(q.codes.cpu().numpy(), ref["codes"])
    if dq:
        assert np.array_equal(q.scale_codes.cpu().numpy(), ref["scale_codes"])
    w_hat = oracle.compute_weight(ref).reshape(N, K)

    Ad, Bd, Xd, dYd = (t.to(DEV) for t in (A, B, X, dY))
    U = torch.empty((M, r), dtype=torch.float32, device=DEV)
    Y = Q.qlora_linear_fwd(q, Ad, Bd, shape.alpha, Xd, U_save=U, check=True)
    dX, dA, dB = Q.qlora_linear_bwd(q, Ad, Bd, shape.alpha, Xd, U, dYd, check=True)
    torch.cuda.synchronize()

    a, b, x, dy = f64(A), f64(B), f64(X), f64(dY)
    rows = slice(None)
    if M > 64:
        rows = np.sort(np.random.default_rng(M).choice(M, 48, replace=False))
        rows = np.concatenate([[0], rows, [M - 1]])
    y_ref, _ = oracle.linear_fwd(w_hat, a, b, shape.alpha, x[rows])
    assert_close(f64(Y)[rows], y_ref, "Y")
    dx_ref, _, _ = oracle.linear_bwd(w_hat, a, b, shape.alpha, x[rows], dy[rows])
    assert_close(f64(dX)[rows], dx_ref, "dX")
    assert_close_scaled(U, oracle.lora_down(a, x), "U")
    da_ref, db_ref = oracle.lora_grads(a, b, shape.alpha, x, dy)
    assert_close_scaled(dA, da_ref, "dA")
    assert_close_scaled(dB, db_ref, "dB")
