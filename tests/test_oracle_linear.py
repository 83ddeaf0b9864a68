"""Pins for the oracle's forward and backward pass (CPU only).

Forward: "LoRA 与 QLoRA：把大模型微调拆成可负担的工程" section 2 and section 3
(zero init of B, merged weight W + (alpha/r) B A); "LoRA 与 QLoRA：用一块 GPU
微调大模型" section "LoRA" (B = 0 gives the original output) and section
"近似" (2dr parameters).  Backward: "QLoRA技术从入门到精通" section 3(3)
(no gradient for W; gradients for A and B only) checked by central finite
differences of the forward pass.
"""

import numpy as np

import oracle


def _rand(rng, *shape, scale=1.0):
    return (rng.standard_normal(shape) * scale).astype(np.float32)


def test_forward_hand_example(golden):
    g = golden("forward_hand_example.txt")
    w = np.array([float(v) for v in g["W"]], np.float32).reshape(2, 2)
    a = np.array([float(v) for v in g["A"]], np.float32).reshape(1, 2)
    b = np.array([float(v) for v in g["B"]], np.float32).reshape(2, 1)
    x = np.array([float(v) for v in g["x"]], np.float32).reshape(1, 2)
    y, _ = oracle.linear_fwd(w, a, b, float(g["alpha"][0]), x)
    assert y.ravel().tolist() == [float(v) for v in g["h"]]


def test_zero_b_gives_the_base_output_exactly():
    rng = np.random.default_rng(0)
    w, a, x = _rand(rng, 24, 64), _rand(rng, 4, 64), _rand(rng, 5, 64)
    b = np.zeros((24, 4), np.float32)
    y, _ = oracle.linear_fwd(w, a, b, 8.0, x)
    assert np.array_equal(y, x.astype(np.float64) @ w.astype(np.float64).T)


def test_merged_weight_identity():
    rng = np.random.default_rng(1)
    w, a, b, x = _rand(rng, 24, 64), _rand(rng, 4, 64), _rand(rng, 24, 4), _rand(rng, 5, 64)
    alpha = 16.0
    y, u = oracle.linear_fwd(w, a, b, alpha, x)
    s = alpha / 4
    merged = w.astype(np.float64) + s * (b.astype(np.float64) @ a.astype(np.float64))
    np.testing.assert_allclose(y, x.astype(np.float64) @ merged.T, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(u, x.astype(np.float64) @ a.astype(np.float64).T, rtol=1e-13)


def test_lora_parameter_count(golden):
    g = golden("storage_bits.txt")
    d, r = int(g["lora_d"][0]), int(g["lora_r"][0])
    a = np.zeros((r, d), np.float32)          # A: r x d_in
    b = np.zeros((d, r), np.float32)          # B: d_out x r
    assert a.size + b.size == int(g["lora_params"][0])
    assert abs((a.size + b.size) / (d * d) - 0.004) < 0.0005


def test_lora_scale_is_alpha_over_r():
    assert oracle.lora_scale(16, 8) == 2.0
    assert oracle.lora_scale(32, 16) == 2.0
    assert oracle.lora_scale(16, 64) == 0.25


def test_backward_matches_central_finite_differences():
    rng = np.random.default_rng(2)
    m, n, k, r, alpha = 3, 8, 64, 2, 5.0
    w = _rand(rng, n, k).astype(np.float64)
    a = _rand(rng, r, k).astype(np.float64)
    b = _rand(rng, n, r).astype(np.float64)
    x = _rand(rng, m, k).astype(np.float64)
    dy = _rand(rng, m, n).astype(np.float64)

    def loss(w_, a_, b_, x_):
        y, _ = oracle.linear_fwd(w_, a_, b_, alpha, x_)
        return float(np.sum(y * dy))

    grads = oracle.linear_bwd(w, a, b, alpha, x, dy)
    assert len(grads) == 3                    # dX, dA, dB; W gets none
    dx, da, db = grads
    h = 1e-3

    def fd(which, arr):
        g = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += h
            minus[idx] -= h
            args_p = dict(w_=w, a_=a, b_=b, x_=x)
            args_m = dict(w_=w, a_=a, b_=b, x_=x)
            args_p[which], args_m[which] = plus, minus
            g[idx] = (loss(**args_p) - loss(**args_m)) / (2 * h)
        return g

    np.testing.assert_allclose(dx, fd("x_", x), rtol=1e-7, atol=1e-8)
    np.testing.assert_allclose(da, fd("a_", a), rtol=1e-7, atol=1e-8)
    np.testing.assert_allclose(db, fd("b_", b), rtol=1e-7, atol=1e-8)


def test_merge_weight_pins():
    rng = np.random.default_rng(4)
    w = (rng.standard_normal((24, 64)) * 0.02).astype(np.float32)
    a, x = _rand(rng, 4, 64), _rand(rng, 5, 64)
    # B = 0: the merged weight is the restored weight itself
    assert np.array_equal(oracle.merge_weight(w, a, np.zeros((24, 4), np.float32), 8.0),
                          w.astype(np.float64))
    # the merged weight reproduces the forward pass of the unmerged layer
    b = _rand(rng, 24, 4, scale=0.1)
    y, _ = oracle.linear_fwd(w, a, b, 8.0, x)
    merged = oracle.merge_weight(w, a, b, 8.0)
    assert np.allclose(x.astype(np.float64) @ merged.T, y, rtol=1e-12, atol=1e-12)
    # the update has rank at most r: removing it from the merged weight gives W back
    assert np.allclose(merged - w, (merged - w) @ np.linalg.pinv(a.astype(np.float64)) @ a,
                       atol=1e-12)
