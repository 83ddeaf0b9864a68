"""Pins for the oracle's level tables (CPU only).

NF4: "QLoRA技术从入门到精通" section 2(3)2) (equal-probability intervals of
N(0,1), the median of each, dense near 0, sparse tails, contains 0) and
"LoRA 与 QLoRA：用一块 GPU 微调大模型" section "量化", part "NF4" (levels at
normal quantiles, exact 0).  Uniform grid: "QLoRA 量化微调" section 7.1.
"""

import numpy as np
from scipy.special import ndtr, ndtri

import oracle


def test_nf4_shape_and_exact_points():
    q = oracle.nf4_levels()
    assert q.dtype == np.float32 and q.shape == (16,)
    assert np.all(np.diff(q) > 0)
    assert q[7] == 0.0 and q[0] == -1.0 and q[15] == 1.0
    assert (q < 0).sum() == 7 and (q > 0).sum() == 8


def test_nf4_dense_near_zero_sparse_in_tails():
    q = oracle.nf4_levels().astype(np.float64)
    pos_gaps = np.diff(q[7:])          # 0 -> +1
    neg_gaps = np.diff(q[:8])[::-1]    # 0 -> -1
    assert np.all(np.diff(pos_gaps) > 0)
    assert np.all(np.diff(neg_gaps) > 0)


def test_nf4_raw_quantiles_match_library_quantile_function():
    neg, pos = oracle.nf4_raw_quantiles()
    ref_pos = ndtri(0.5 + (np.arange(1, 9) - 0.5) / 16.0)
    ref_neg = ndtri(0.5 - (np.arange(1, 8) - 0.5) / 14.0)
    np.testing.assert_allclose(pos, ref_pos, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(neg, ref_neg, rtol=1e-13, atol=1e-15)
    ref_levels = np.concatenate([(ref_neg / -ref_neg[-1])[::-1], [0.0],
                                 ref_pos / ref_pos[-1]]).astype(np.float32)
    assert np.array_equal(oracle.nf4_levels().view(np.uint32), ref_levels.view(np.uint32))


def test_nf4_levels_are_interval_medians_of_equal_mass():
    neg, pos = oracle.nf4_raw_quantiles()
    # positive half: 8 intervals of mass 1/16 with boundaries b_j
    b = np.concatenate([[0.0], ndtri(0.5 + np.arange(1, 8) / 16.0), [np.inf]])
    for j in range(8):
        lo, hi = ndtr(b[j]), ndtr(b[j + 1])
        assert abs((hi - lo) - 1.0 / 16.0) < 1e-12
        assert abs((ndtr(pos[j]) - lo) - (hi - ndtr(pos[j]))) < 1e-12
    # negative half: 7 intervals of mass 1/14
    b = np.concatenate([[0.0], ndtri(0.5 - np.arange(1, 7) / 14.0), [-np.inf]])
    for j in range(7):
        hi, lo = ndtr(b[j]), ndtr(b[j + 1])
        assert abs((hi - lo) - 1.0 / 14.0) < 1e-12
        assert abs((hi - ndtr(neg[j])) - (ndtr(neg[j]) - lo)) < 1e-12


def test_uniform_grid_points_printed_on_page(golden):
    g = golden("worked_example_uniform.txt")
    q = oracle.uniform_levels()
    assert q[0] == -1.0 and q[15] == 1.0
    assert q[int(g["index_0"][0])] == np.float32(float(g["level_0"][0]))
    np.testing.assert_allclose(np.diff(q.astype(np.float64)), 2.0 / 15.0, rtol=1e-6)


def test_bf16_rounding_matches_library_conversion():
    import torch
    rng = np.random.default_rng(11)
    x = np.concatenate([rng.standard_normal(20000).astype(np.float32) * 10.0 ** rng.integers(-6, 6, 20000),
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 0.0, -0.0,
                                  3.4e38, 1e-40], np.float32)]).astype(np.float32)
    ref = torch.from_numpy(x).bfloat16().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.f32_to_bf16_bits(x), ref)
    # ties go to even: 1 + 2^-8 is halfway between 1 and 1 + 2^-7
    assert oracle.round_to_bf16(np.float32(1.0 + 2 ** -8)) == np.float32(1.0)
    assert oracle.round_to_bf16(np.float32(1.0 + 3 * 2 ** -8)) == np.float32(1.0 + 2 ** -6)
