"""Pins for the LoRA-dropout oracle (CPU only): the bit layout of the keep
mask, the special cases (keep everything, drop everything), the gradients
against central differences, and the unbiasedness of inverted dropout."""

import numpy as np

import oracle


def test_mask_bit_layout():
    m = np.array([[0b10110001, 0x00], [0xFF, 0b00000010]], dtype=np.uint8)
    d = oracle.unpack_keep_mask(m, 16)
    assert d[0, :8].tolist() == [1, 0, 0, 0, 1, 1, 0, 1]
    assert not d[0, 8:].any() and d[1, :8].all()
    assert d[1, 8:].tolist() == [0, 1, 0, 0, 0, 0, 0, 0]


def _case(M=6, N=5, K=16, r=3, seed=0):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((N, K)), rng.standard_normal((r, K)), rng.standard_normal((N, r)),
            rng.standard_normal((M, K)), rng.standard_normal((M, N)),
            rng.integers(0, 256, (M, K // 8)).astype(np.uint8))


def test_keep_all_is_the_plain_layer():
    w, a, b, x, dy, _ = _case()
    ones = np.full((6, 2), 0xFF, np.uint8)
    y, u = oracle.linear_fwd_dropout(w, a, b, 6.0, 0.0, ones, x)
    y1, u1 = oracle.linear_fwd(w, a, b, 6.0, x)
    assert np.allclose(y, y1, rtol=1e-13) and np.allclose(u, u1, rtol=1e-13)
    g = oracle.linear_bwd_dropout(w, a, b, 6.0, 0.0, ones, x, dy)
    g1 = oracle.linear_bwd(w, a, b, 6.0, x, dy)
    for p, q in zip(g, g1):
        assert np.allclose(p, q, rtol=1e-13, atol=1e-13)


def test_drop_all_is_the_base_layer():
    w, a, b, x, dy, _ = _case()
    zeros = np.zeros((6, 2), np.uint8)
    y, u = oracle.linear_fwd_dropout(w, a, b, 6.0, 0.3, zeros, x)
    assert np.array_equal(y, x @ w.T) and not u.any()
    dx, da, db = oracle.linear_bwd_dropout(w, a, b, 6.0, 0.3, zeros, x, dy)
    assert np.array_equal(dx, dy @ w) and not da.any() and not db.any()


def test_gradients_are_the_loss_derivatives():
    w, a, b, x, g, mask = _case(seed=4)
    p = 0.25
    loss = lambda a_, b_, x_: float((oracle.linear_fwd_dropout(w, a_, b_, 6.0, p, mask, x_)[0] * g).sum())
    dx, da, db = oracle.linear_bwd_dropout(w, a, b, 6.0, p, mask, x, g)
    h = 1e-6
    for idx in ((0, 0), (2, 11), (1, 7)):
        ap, am = a.copy(), a.copy()
        ap[idx] += h; am[idx] -= h
        fd = (loss(ap, b, x) - loss(am, b, x)) / (2 * h)
        assert abs(fd - da[idx]) < 1e-6 * (1 + abs(fd))
    for idx in ((0, 1), (4, 2)):
        bp, bm = b.copy(), b.copy()
        bp[idx] += h; bm[idx] -= h
        fd = (loss(a, bp, x) - loss(a, bm, x)) / (2 * h)
        assert abs(fd - db[idx]) < 1e-6 * (1 + abs(fd))
    d = oracle.unpack_keep_mask(mask, 16)
    picked = [(0, 0), (3, 9), (5, 15)]
    picked += [tuple(np.argwhere(d == 0)[0]), tuple(np.argwhere(d == 1)[0])]
    for idx in picked:
        xp, xm = x.copy(), x.copy()
        xp[idx] += h; xm[idx] -= h
        fd = (loss(a, b, xp) - loss(a, b, xm)) / (2 * h)
        assert abs(fd - dx[idx]) < 1e-6 * (1 + abs(fd))


def test_inverted_dropout_is_unbiased():
    # the mean of U over many masks (keep probability 1 - p) is X A^T
    w, a, b, x, _, _ = _case(M=2, K=16, seed=2)
    rng = np.random.default_rng(3)
    p, n = 0.3, 20000
    keep = rng.random((n, 2, 16)) >= p
    packed = np.packbits(keep, axis=-1, bitorder="little")
    acc = np.zeros((2, 3))
    for i in range(n):
        acc += oracle.linear_fwd_dropout(w, a, b, 6.0, p, packed[i], x)[1]
    mean = acc / n
    ref = x @ a.T
    se = np.sqrt(p / (1 - p) * (x * x) @ (a * a).T / n)   # standard error of each mean
    assert np.all(np.abs(mean - ref) < 5 * se)


def test_binding_mask_packing_matches_the_oracle_layout():
    # the binding's keep-mask helper (torch's generator, any device) packs bit
    # k % 8 of byte [m][k // 8]; the oracle unpacks it back to the draw
    import torch

    from bit_nf4_quantized_17_b200 import qlora as Q

    g = torch.Generator().manual_seed(3)
    m = Q.dropout_keep_mask(4, 64, 0.3, generator=g, device="cpu")
    g2 = torch.Generator().manual_seed(3)
    keep = (torch.rand((4, 8, 8), generator=g2) >= 0.3).reshape(4, 64).numpy()
    assert m.shape == (4, 8) and m.dtype == torch.uint8
    assert np.array_equal(oracle.unpack_keep_mask(m.numpy(), 64), keep.astype(np.float64))
