"""GPU parity of LoRA dropout on the adapter input (qlora_linear_fwd_ex /
_bwd_ex) against the oracle, on every path of the library; the dropped-out
copy X (.) D is compared bit for bit, the outputs within the stated
tolerance.  One case combines dropout with several adapters per batch."""

import numpy as np
import pytest
import torch

import oracle
from bit_nf4_quantized_17_b200 import qlora as Q
from bit_nf4_quantized_17_b200 import workloads as WL
from parity import assert_close, assert_close_scaled, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = [  # M, N, K, r, p
    (1, 1024, 2048, 16, 0.1),
    (2, 512, 1024, 8, 0.05),
    (13, 1024, 2048, 64, 0.1),
    (700, 512, 2048, 16, 0.2),
    (4096, 2048, 1024, 16, 0.1),
]


def _mask(M, K, p, seed):
    keep = np.random.default_rng(seed).random((M, K)) >= p
    return np.packbits(keep.reshape(M, K // 8, 8), axis=-1, bitorder="little").reshape(M, K // 8)


@pytest.mark.parametrize("M,N,K,r,p", CASES, ids=["m1", "m2", "m13", "m700", "m4096"])
def test_dropout_against_oracle(M, N, K, r, p):
    shape = WL.LinearShape(N, K, r, 2.0 * r)
    inp = WL.linear_inputs(shape, M, 50 + M)
    inp["B"] = WL.randn((N, r), 0.05, 51 + M, torch.bfloat16)
    W, A, B, X, dY = (inp[k] for k in ("W", "A", "B", "X", "dY"))
    mask = _mask(M, K, p, M)
    q = Q.qlora_quantize(W.to(DEV))
    Ad, Bd, Xd, dYd = (t.to(DEV) for t in (A, B, X, dY))
    md = torch.from_numpy(mask).to(DEV)
    xdrop = torch.empty_like(Xd)
    U = torch.empty((M, r), dtype=torch.float32, device=DEV)
    Y = Q.qlora_linear_fwd_ex(q, Ad, Bd, r, shape.alpha, Xd, p=p, keep_mask=md, x_drop=xdrop,
                              U_save=U, check=True)
    dX, dA, dB = Q.qlora_linear_bwd_ex(q, Ad, Bd, r, shape.alpha, Xd, U, dYd, p=p, keep_mask=md,
                                       x_drop=xdrop, check=True)
    torch.cuda.synchronize()

    d = oracle.unpack_keep_mask(mask, K)
    xb = X.view(torch.int16).numpy()
    assert np.array_equal(xdrop.cpu().view(torch.int16).numpy(), np.where(d > 0, xb, 0))
    w_hat = oracle.compute_weight(oracle.quantize(W.float().numpy(), 64, 256)).reshape(N, K)
    a, b, x, dy = f64(A), f64(B), f64(X), f64(dY)
    rows = np.arange(M)
    if M > 64:
        rows = np.unique(np.concatenate([[0, M - 1], np.random.default_rng(M).choice(M, 48, replace=False)]))
    y_ref, _ = oracle.linear_fwd_dropout(w_hat, a, b, shape.alpha, p, mask[rows], x[rows])
    assert_close(f64(Y)[rows], y_ref, "Y")
    dx_ref, _, _ = oracle.linear_bwd_dropout(w_hat, a, b, shape.alpha, p, mask[rows], x[rows], dy[rows])
    assert_close(f64(dX)[rows], dx_ref, "dX")
    _, u_ref = oracle.linear_fwd_dropout(w_hat, a, b, shape.alpha, p, mask, x)
    assert_close_scaled(U, u_ref, "U")
    _, da_ref, db_ref = oracle.linear_bwd_dropout(w_hat, a, b, shape.alpha, p, mask, x, dy)
    assert_close_scaled(dA, da_ref, "dA")
    assert_close_scaled(dB, db_ref, "dB")


def test_dropout_with_several_adapters():
    # dropout and per-token adapters together: per adapter, the dropout oracle
    # on that adapter's tokens; dX of adapter-less tokens is the base product
    M, N, K, r, n, p = 300, 1024, 2048, 16, 3, 0.1
    shape = WL.LinearShape(N, K, n * r, 2.0 * r)
    inp = WL.linear_inputs(shape, M, 77)
    W, X, dY = inp["W"], inp["X"], inp["dY"]
    As = [WL.randn((r, K), 0.25, 80 + a, torch.bfloat16) for a in range(n)]
    Bs = [WL.randn((N, r), 0.05, 90 + a, torch.bfloat16) for a in range(n)]
    ids = np.random.default_rng(1).integers(-1, n, M).astype(np.int32)
    mask = _mask(M, K, p, 2)
    q = Q.qlora_quantize(W.to(DEV))
    A, B = torch.cat(As, 0).to(DEV), torch.cat(Bs, 1).contiguous().to(DEV)
    Xd, dYd = X.to(DEV), dY.to(DEV)
    idd, md = torch.from_numpy(ids).to(DEV), torch.from_numpy(mask).to(DEV)
    xdrop = torch.empty_like(Xd)
    U = torch.empty((M, n * r), dtype=torch.float32, device=DEV)
    Y = Q.qlora_linear_fwd_ex(q, A, B, r, 2.0 * r, Xd, adapter=idd, p=p, keep_mask=md,
                              x_drop=xdrop, U_save=U, check=True)
    dX, dA, dB = Q.qlora_linear_bwd_ex(q, A, B, r, 2.0 * r, Xd, U, dYd, adapter=idd, p=p,
                                       keep_mask=md, x_drop=xdrop, check=True)
    torch.cuda.synchronize()
    w_hat = oracle.compute_weight(oracle.quantize(W.float().numpy(), 64, 256)).reshape(N, K)
    x, dy = f64(X), f64(dY)
    y_ref = x @ w_hat.T
    dx_ref = dy @ w_hat
    da_ref = np.zeros((n * r, K))
    db_ref = np.zeros((N, n * r))
    for a in range(n):
        rows = np.nonzero(ids == a)[0]
        ya, _ = oracle.linear_fwd_dropout(w_hat, f64(As[a]), f64(Bs[a]), 2.0 * r, p, mask[rows], x[rows])
        y_ref[rows] = ya
        dxa, daa, dba = oracle.linear_bwd_dropout(w_hat, f64(As[a]), f64(Bs[a]), 2.0 * r, p,
                                                  mask[rows], x[rows], dy[rows])
        dx_ref[rows] = dxa
        da_ref[a * r:(a + 1) * r] = daa
        db_ref[:, a * r:(a + 1) * r] = dba
    assert_close(f64(Y), y_ref, "Y")
    assert_close(f64(dX), dx_ref, "dX")
    assert_close_scaled(dA, da_ref, "dA")
    assert_close_scaled(dB, db_ref, "dB")


def test_keep_mask_helper_rate():
    m = Q.dropout_keep_mask(512, 4096, 0.1, generator=torch.Generator(DEV).manual_seed(0))
    assert m.shape == (512, 512) and m.dtype == torch.uint8
    kept = int(np.unpackbits(m.cpu().numpy(), bitorder="little").sum())
    frac = kept / (512 * 4096)
    assert abs(frac - 0.9) < 0.005


@pytest.mark.parametrize("M", [13, 700])
def test_recomputed_u_matches_the_saved_one(M):
    # the backward without U recomputes it from X (.) D with the same scale and
    # adapter mask as the forward: the gradients are bit-identical
    N, K, r, n, p = 512, 1024, 8, 2, 0.1
    shape = WL.LinearShape(N, K, n * r, 2.0 * r)
    inp = WL.linear_inputs(shape, M, 300 + M)
    q = Q.qlora_quantize(inp["W"].to(DEV))
    A = WL.randn((n * r, K), 0.3, 5, torch.bfloat16).to(DEV)
    B = WL.randn((N, n * r), 0.05, 6, torch.bfloat16).to(DEV)
    X, dY = inp["X"].to(DEV), inp["dY"].to(DEV)
    ids = torch.from_numpy(np.random.default_rng(M).integers(-1, n, M).astype(np.int32)).to(DEV)
    md = torch.from_numpy(_mask(M, K, p, 9)).to(DEV)
    xdrop = torch.empty_like(X)
    U = torch.empty((M, n * r), dtype=torch.float32, device=DEV)
    Q.qlora_linear_fwd_ex(q, A, B, r, 2.0 * r, X, adapter=ids, p=p, keep_mask=md, x_drop=xdrop,
                          U_save=U, check=True)
    g_saved = Q.qlora_linear_bwd_ex(q, A, B, r, 2.0 * r, X, U, dY, adapter=ids, p=p,
                                    keep_mask=md, x_drop=xdrop, check=True)
    g_recomp = Q.qlora_linear_bwd_ex(q, A, B, r, 2.0 * r, X, None, dY, adapter=ids, p=p,
                                     keep_mask=md, x_drop=xdrop, check=True)
    torch.cuda.synchronize()
    for a, b, name in zip(g_saved, g_recomp, ("dX", "dA", "dB")):
        assert torch.equal(a, b), name
