"""Pins for the multi-adapter oracle (CPU only).

Each pin holds for any correct implementation and fails for the plausible
mistakes: a token given another adapter's pair, an adapter's gradient picking
up other tokens, the scale taken from the stacked rank, a transposed operand.
"""

import numpy as np

import oracle


def _case(M=12, N=10, K=9, r=3, n=3, seed=0):
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((N, K))
    As = [rng.standard_normal((r, K)) for _ in range(n)]
    Bs = [rng.standard_normal((N, r)) for _ in range(n)]
    x = rng.standard_normal((M, K))
    dy = rng.standard_normal((M, N))
    ids = rng.integers(-1, n, M)
    return w, As, Bs, x, dy, ids


def test_one_adapter_for_every_token_is_the_single_layer():
    w, As, Bs, x, dy, _ = _case(n=1)
    ids = np.zeros(len(x), dtype=np.int64)
    y, u = oracle.linear_fwd_multi(w, As, Bs, 6.0, x, ids)
    y1, u1 = oracle.linear_fwd(w, As[0], Bs[0], 6.0, x)
    assert np.allclose(y, y1, rtol=1e-13, atol=1e-13) and np.allclose(u, u1, rtol=1e-13)
    dx, da, db = oracle.linear_bwd_multi(w, As, Bs, 6.0, x, dy, ids)
    dx1, da1, db1 = oracle.linear_bwd(w, As[0], Bs[0], 6.0, x, dy)
    for p, q in ((dx, dx1), (da, da1), (db, db1)):
        assert np.allclose(p, q, rtol=1e-13, atol=1e-13)


def test_no_adapter_is_the_base_layer():
    w, As, Bs, x, dy, _ = _case()
    ids = -np.ones(len(x), dtype=np.int64)
    y, u = oracle.linear_fwd_multi(w, As, Bs, 6.0, x, ids)
    assert np.array_equal(y, x @ w.T) and not u.any()
    dx, da, db = oracle.linear_bwd_multi(w, As, Bs, 6.0, x, dy, ids)
    assert np.array_equal(dx, dy @ w) and not da.any() and not db.any()


def test_each_token_brute_force():
    # element by element: y[m][n] = sum_k x w + s sum_j (sum_k x A_a) B_a
    w, As, Bs, x, dy, ids = _case(M=6, N=4, K=5, r=2, n=2, seed=3)
    s = 8.0 / 2
    y, u = oracle.linear_fwd_multi(w, As, Bs, 8.0, x, ids)
    for m in range(6):
        a = ids[m]
        for n_ in range(4):
            ref = sum(x[m, k] * w[n_, k] for k in range(5))
            if 0 <= a < 2:
                for j in range(2):
                    uj = sum(x[m, k] * As[a][j, k] for k in range(5))
                    ref += s * uj * Bs[a][n_, j]
            assert abs(y[m, n_] - ref) < 1e-12
        for c in range(4):
            want = sum(x[m, k] * As[c // 2][c % 2, k] for k in range(5)) if c // 2 == a else 0.0
            assert abs(u[m, c] - want) < 1e-12


def test_gradients_are_the_loss_derivatives():
    # L = sum(Y * G): central differences in A_a, B_a and X, for every adapter
    w, As, Bs, x, g, ids = _case(M=7, N=5, K=4, r=2, n=3, seed=5)
    ids[:3] = [0, 1, 2]
    loss = lambda As_, Bs_, x_: float((oracle.linear_fwd_multi(w, As_, Bs_, 3.0, x_, ids)[0] * g).sum())
    dx, da, db = oracle.linear_bwd_multi(w, As, Bs, 3.0, x, g, ids)
    h = 1e-6
    for a in range(3):
        for (j, k) in ((0, 0), (1, 3)):
            Ap = [t.copy() for t in As]; Am = [t.copy() for t in As]
            Ap[a][j, k] += h; Am[a][j, k] -= h
            fd = (loss(Ap, Bs, x) - loss(Am, Bs, x)) / (2 * h)
            assert abs(fd - da[a * 2 + j, k]) < 1e-6 * (1 + abs(fd))
        for (n_, j) in ((0, 1), (4, 0)):
            Bp = [t.copy() for t in Bs]; Bm = [t.copy() for t in Bs]
            Bp[a][n_, j] += h; Bm[a][n_, j] -= h
            fd = (loss(As, Bp, x) - loss(As, Bm, x)) / (2 * h)
            assert abs(fd - db[n_, a * 2 + j]) < 1e-6 * (1 + abs(fd))
    for (m, k) in ((0, 1), (2, 3), (6, 0)):
        xp, xm = x.copy(), x.copy()
        xp[m, k] += h; xm[m, k] -= h
        fd = (loss(As, Bs, xp) - loss(As, Bs, xm)) / (2 * h)
        assert abs(fd - dx[m, k]) < 1e-6 * (1 + abs(fd))


def test_token_order_does_not_matter():
    w, As, Bs, x, dy, ids = _case(seed=9)
    p = np.random.default_rng(1).permutation(len(x))
    y, u = oracle.linear_fwd_multi(w, As, Bs, 6.0, x, ids)
    yp, up = oracle.linear_fwd_multi(w, As, Bs, 6.0, x[p], ids[p])
    assert np.allclose(yp, y[p], rtol=1e-13) and np.allclose(up, u[p], rtol=1e-13)
    dx, da, db = oracle.linear_bwd_multi(w, As, Bs, 6.0, x, dy, ids)
    dxp, dap, dbp = oracle.linear_bwd_multi(w, As, Bs, 6.0, x[p], dy[p], ids[p])
    assert np.allclose(dxp, dx[p], rtol=1e-12, atol=1e-12)
    assert np.allclose(dap, da, rtol=1e-12, atol=1e-12) and np.allclose(dbp, db, rtol=1e-12, atol=1e-12)
