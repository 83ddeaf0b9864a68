"""Pins for the oracle's AdamW step (CPU only).

AdamW (Adam with decoupled weight decay, Loshchilov and Hutter) is the
optimiser of the adapters; the pins are its closed forms."""

import numpy as np

import oracle


def test_first_step_is_normalised_gradient():
    # zero state, step 1: m^ = g, v^ = g^2, so the update is lr g / (|g| + eps)
    rng = np.random.default_rng(0)
    p, g = rng.standard_normal(1000), rng.standard_normal(1000)
    z = np.zeros(1000)
    p1, m1, v1 = oracle.adamw_step(p, g, z, z, 1, lr=1e-3, eps=1e-8)
    assert np.allclose(p1, p - 1e-3 * g / (np.abs(g) + 1e-8), rtol=1e-14, atol=1e-17)
    assert np.allclose(m1, 0.1 * g) and np.allclose(v1, 0.001 * g * g)


def test_zero_gradient_only_decays():
    # g = 0 with zero moments: p <- p (1 - lr wd), step after step
    p = np.linspace(-2, 2, 101)
    z = np.zeros_like(p)
    q, m, v = p, z, z
    for t in range(1, 6):
        q, m, v = oracle.adamw_step(q, z, m, v, t, lr=0.01, weight_decay=0.1)
    assert np.allclose(q, p * (1 - 0.01 * 0.1) ** 5, rtol=1e-14)


def test_recurrence_against_a_loop():
    # three steps against an element-by-element restatement of the moments
    rng = np.random.default_rng(1)
    p = rng.standard_normal(7)
    gs = [rng.standard_normal(7) for _ in range(3)]
    m = np.zeros(7)
    v = np.zeros(7)
    q = p.copy()
    for t, g in enumerate(gs, start=1):
        q, m, v = oracle.adamw_step(q, g, m, v, t, lr=0.05, beta1=0.8, beta2=0.9,
                                    eps=1e-6, weight_decay=0.01, grad_scale=0.5)
    ref = p.copy()
    for i in range(7):
        mi = vi = 0.0
        pi = p[i]
        for t, g in enumerate(gs, start=1):
            gi = 0.5 * g[i]
            mi = 0.8 * mi + 0.2 * gi
            vi = 0.9 * vi + 0.1 * gi * gi
            pi = pi - 0.05 * ((mi / (1 - 0.8 ** t)) / (np.sqrt(vi / (1 - 0.9 ** t)) + 1e-6) + 0.01 * pi)
        ref[i] = pi
    assert np.allclose(q, ref, rtol=1e-13)
