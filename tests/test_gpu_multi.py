"""GPU parity of several adapters over one NF4 base (one adapter per token).

The adapters are stacked along the rank (A: (n r) x d_in, B: d_out x (n r)),
token m uses adapter ids[m] (-1: none).  Against the oracle's per-adapter
restatement: Y and dX (bf16) within the stated tolerance, U, dA and dB (fp32)
within the same bar in their own scale, and the entries that must be zero
(other adapters' U columns, gradients of adapters no token uses) exactly zero.
Every path of the library: decode forward (W in tensor memory) with the dX
GEMV, the small-batch tensor-core path, the split-K single-CTA kernel and
the CTA-pair kernels.
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

CASES = [  # M, N, K, n adapters, r
    (1, 1024, 2048, 4, 16),
    (2, 512, 1024, 3, 8),
    (13, 1024, 2048, 4, 16),
    (700, 512, 2048, 2, 64),
    (4096, 2048, 1024, 8, 16),
]


@pytest.mark.parametrize("M,N,K,n,r", CASES, ids=["m1", "m2", "m13", "m700", "m4096"])
def test_multi_adapter_against_oracle(M, N, K, n, r):
    seed = M + 7 * n
    shape = WL.LinearShape(N, K, n * r, 2.0 * r)
    inp = WL.linear_inputs(shape, M, seed)
    W, X, dY = inp["W"], inp["X"], inp["dY"]
    As = [WL.randn((r, K), 1.0 / np.sqrt(r), seed + 10 + a, torch.bfloat16) for a in range(n)]
    Bs = [WL.randn((N, r), 0.05, seed + 40 + a, torch.bfloat16) for a in range(n)]
    A = torch.cat(As, 0)
    B = torch.cat(Bs, 1).contiguous()
    rng = np.random.default_rng(seed)
    ids = rng.integers(-1, n, M).astype(np.int32)
    if M >= n:
        ids[:n] = np.arange(n)          # every adapter has a token ...
    if n > 2 and M > 2 * n:
        ids[ids == n - 1] = 0           # ... except the last one, in the large cases
    alpha = 2.0 * r

    q = Q.qlora_quantize(W.to(DEV))
    Ad, Bd, Xd, dYd = (t.to(DEV) for t in (A, B, X, dY))
    idd = torch.from_numpy(ids).to(DEV)
    U = torch.empty((M, n * r), dtype=torch.float32, device=DEV)
    Y = Q.qlora_linear_fwd_multi(q, Ad, Bd, r, alpha, idd, Xd, U_save=U, check=True)
    dX, dA, dB = Q.qlora_linear_bwd_multi(q, Ad, Bd, r, alpha, idd, Xd, U, dYd, check=True)
    torch.cuda.synchronize()

    w_hat = oracle.compute_weight(oracle.quantize(W.float().numpy(), 64, 256)).reshape(N, K)
    a_l, b_l = [f64(t) for t in As], [f64(t) for t in Bs]
    x, dy = f64(X), f64(dY)
    rows = np.arange(M)
    if M > 64:
        rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, 48, replace=False)]))
    y_ref, _ = oracle.linear_fwd_multi(w_hat, a_l, b_l, alpha, x[rows], ids[rows])
    assert_close(f64(Y)[rows], y_ref, "Y")
    dx_ref, _, _ = oracle.linear_bwd_multi(w_hat, a_l, b_l, alpha, x[rows], dy[rows], ids[rows])
    assert_close(f64(dX)[rows], dx_ref, "dX")
    _, u_ref = oracle.linear_fwd_multi(w_hat, a_l, b_l, alpha, x, ids)
    assert_close_scaled(U, u_ref, "U")
    u = U.cpu().numpy()
    own = (np.arange(n * r)[None, :] // r) == ids[:, None]
    assert not u[~own].any(), "U has values outside each token's adapter columns"
    _, da_ref, db_ref = oracle.linear_bwd_multi(w_hat, a_l, b_l, alpha, x, dy, ids)
    assert_close_scaled(dA, da_ref, "dA")
    assert_close_scaled(dB, db_ref, "dB")
    used = set(ids[(ids >= 0) & (ids < n)].tolist())
    for a in range(n):
        if a not in used:
            assert not dA[a * r:(a + 1) * r].any() and not dB[:, a * r:(a + 1) * r].any()


def test_multi_with_one_adapter_is_the_single_layer():
    # n = 1 and every token on adapter 0: bit-identical to qlora_linear_fwd / _bwd
    shape = WL.LinearShape(1024, 2048, 16, 32.0)
    inp = WL.linear_inputs(shape, 300, 5)
    q = Q.qlora_quantize(inp["W"].to(DEV))
    A, B, X, dY = (inp[k].to(DEV) for k in ("A", "B", "X", "dY"))
    ids = torch.zeros(300, dtype=torch.int32, device=DEV)
    U1 = torch.empty((300, 16), dtype=torch.float32, device=DEV)
    U2 = torch.empty_like(U1)
    Y1 = Q.qlora_linear_fwd(q, A, B, 32.0, X, U_save=U1)
    Y2 = Q.qlora_linear_fwd_multi(q, A, B, 16, 32.0, ids, X, U_save=U2)
    g1 = Q.qlora_linear_bwd(q, A, B, 32.0, X, U1, dY)
    g2 = Q.qlora_linear_bwd_multi(q, A, B, 16, 32.0, ids, X, U2, dY)
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2) and torch.equal(U1, U2)
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)


def test_multi_argument_errors():
    q = Q.qlora_quantize(torch.randn(256, 256, device=DEV, dtype=torch.bfloat16))
    X = torch.zeros((4, 256), dtype=torch.bfloat16, device=DEV)
    ids = torch.zeros(4, dtype=torch.int32, device=DEV)

    def ab(rows):
        return (torch.zeros((rows, 256), dtype=torch.bfloat16, device=DEV),
                torch.zeros((256, rows), dtype=torch.bfloat16, device=DEV))

    with pytest.raises(ValueError):          # 24 rows are not whole rank-5 adapters
        Q.qlora_linear_fwd_multi(q, *ab(24), 5, 8.0, ids, X)
    with pytest.raises(Q.QloraError) as e:   # 3 x 5 = 15 stacked ranks: not a multiple of 8
        Q.qlora_linear_fwd_multi(q, *ab(15), 5, 8.0, ids, X)
    assert e.value.status == Q.QLORA_ERR_UNSUPPORTED
    with pytest.raises(Q.QloraError) as e:   # 33 x 8 = 264 > 256
        Q.qlora_linear_fwd_multi(q, *ab(264), 8, 8.0, ids, X)
    assert e.value.status == Q.QLORA_ERR_SHAPE
