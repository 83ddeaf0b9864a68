"""Pins for the oracle's quantiser, double quantisation and dequantiser.

Sources: "QLoRA技术从入门到精通" section 3(1)/3(2); "LoRA 与 QLoRA：用一块
GPU 微调大模型" section "量化"; "QLoRA 量化微调" section 7.1 (worked example,
storage arithmetic).
"""

from fractions import Fraction

import numpy as np
import pytest

import oracle


def _exact_nearest(x, levels):
    """Brute force: argmin_k |x - q_k| in exact rational arithmetic, ties low."""
    xf = Fraction(float(x))
    d = [abs(xf - Fraction(float(q))) for q in levels]
    best = min(d)
    return d.index(best)


# ---------------------------------------------------------- worked example

def test_worked_example_uniform_grid(golden):
    g = golden("worked_example_uniform.txt")
    group = np.array([float(v) for v in g["group"]], dtype=np.float32)
    qt = oracle.quantize(group, blocksize=4, dq_blocksize=0,
                         levels=oracle.uniform_levels())
    assert qt["absmax"][0] == np.float32(float(g["absmax"][0]))
    x0 = group[0] / qt["absmax"][0]
    assert abs(float(x0) - float(g["normalised_0"][0])) < 1e-4
    assert int(qt["idx"][0]) == int(g["index_0"][0])
    assert format(int(qt["idx"][0]), "04b") == g["index_0_binary"][0]
    assert [int(v) for v in qt["idx"]] == [int(v) for v in g["index_all"]]
    w_hat = oracle.dequantize(qt)
    assert abs(float(w_hat[0]) - float(g["dequantised_0"][0])) < 1e-6
    assert abs(abs(float(w_hat[0]) - float(group[0])) - float(g["abs_error_0"][0])) < 1e-6


# ------------------------------------------------------------ nearest level

@pytest.mark.parametrize("table", ["nf4", "uniform"])
def test_nearest_level_matches_brute_force_random(table):
    levels = oracle.nf4_levels() if table == "nf4" else oracle.uniform_levels()
    rng = np.random.default_rng(7)
    x = rng.uniform(-1.0, 1.0, 200_000).astype(np.float32)
    got = oracle.nearest_level(x, levels)
    d = np.abs(x.astype(np.float64)[:, None] - levels.astype(np.float64)[None, :])
    ref = np.argmin(d, axis=1)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("table", ["nf4", "uniform"])
def test_nearest_level_at_and_around_every_midpoint(table):
    levels = oracle.nf4_levels() if table == "nf4" else oracle.uniform_levels()
    pts = []
    for k in range(15):
        m = np.float32((np.float64(levels[k]) + np.float64(levels[k + 1])) / 2)
        for steps in range(-3, 4):
            v = m
            for _ in range(abs(steps)):
                v = np.nextafter(v, np.float32(np.inf if steps > 0 else -np.inf))
            pts.append(v)
    pts += [np.float32(v) for v in (-1.0, 1.0, 0.0, -0.0, 1e-30, -1e-30, 1e-45)]
    pts = np.array(pts, dtype=np.float32)
    got = oracle.nearest_level(pts, levels)
    ref = [_exact_nearest(v, levels) for v in pts]
    assert list(got) == ref


def test_nearest_level_error_is_at_most_half_the_local_gap():
    levels = oracle.nf4_levels().astype(np.float64)
    x = np.linspace(-1, 1, 100_001, dtype=np.float32)
    idx = oracle.nearest_level(x, levels.astype(np.float32)).astype(np.int64)
    err = np.abs(x.astype(np.float64) - levels[idx])
    gaps = np.diff(levels)
    lo_gap = np.where(idx > 0, gaps[np.maximum(idx - 1, 0)], 0.0)
    hi_gap = np.where(idx < 15, gaps[np.minimum(idx, 14)], 0.0)
    assert np.all(err <= np.maximum(lo_gap, hi_gap) / 2 + 1e-7)


# ---------------------------------------------------------------- packing

def test_pack_nibble_order_and_round_trip():
    assert oracle.pack_nibbles(np.array([1, 2], np.uint8))[0] == 0x21
    rng = np.random.default_rng(1)
    idx = rng.integers(0, 16, 1001).astype(np.uint8)
    codes = oracle.pack_nibbles(idx)
    assert codes.size == 501 and (codes[-1] >> 4) == 0
    assert np.array_equal(oracle.unpack_nibbles(codes, 1001), idx)


def test_block_absmax_brute_force_with_partial_tail():
    rng = np.random.default_rng(2)
    w = rng.standard_normal(64 * 3 + 5).astype(np.float32)
    s = oracle.block_absmax(w, 64)
    assert s.size == 4
    for b in range(4):
        assert s[b] == max(abs(float(v)) for v in w[64 * b:64 * b + 64])


# ------------------------------------------------------------- round trip

@pytest.mark.parametrize("table", ["nf4", "uniform"])
def test_on_grid_weights_round_trip_exactly_without_dq(table):
    levels = oracle.nf4_levels() if table == "nf4" else oracle.uniform_levels()
    rng = np.random.default_rng(3)
    nb = 40
    idx = rng.integers(0, 16, (nb, 64)).astype(np.uint8)
    idx[:, 5] = 15                                    # absmax element: level +1
    scale = (2.0 ** rng.integers(-12, 3, nb)).astype(np.float32)
    w = (levels[idx] * scale[:, None]).astype(np.float32).ravel()
    qt = oracle.quantize(w, 64, 0, levels)
    assert np.array_equal(qt["idx"], idx.ravel())
    assert np.array_equal(oracle.dequantize(qt).view(np.uint32), w.view(np.uint32))


def test_on_grid_weights_round_trip_exactly_with_dq_and_one_shared_scale():
    levels = oracle.nf4_levels()
    rng = np.random.default_rng(4)
    nb = 600
    idx = rng.integers(0, 16, (nb, 64)).astype(np.uint8)
    idx[:, 0] = 0                                     # absmax element: level -1
    w = (levels[idx] * np.float32(0.03125)).astype(np.float32).ravel()
    qt = oracle.quantize(w, 64, 256, levels)
    assert qt["mean"] == np.float32(0.03125)
    assert np.all(qt["scale_codes"] == 0) and np.all(qt["factors"] == 0)
    assert np.array_equal(oracle.dequantize(qt).view(np.uint32), w.view(np.uint32))


def test_zero_block_maps_to_zero_level():
    w = np.zeros(128, np.float32)
    w[64:] = np.linspace(-1, 1, 64, dtype=np.float32)
    qt = oracle.quantize(w, 64, 256)
    assert np.all(qt["idx"][:64] == 7)
    assert np.all(oracle.dequantize(qt)[:64] == 0.0)


def test_non_finite_weight_is_rejected():
    w = np.ones(64, np.float32)
    w[3] = np.nan
    with pytest.raises(ValueError):
        oracle.quantize(w)
    w[3] = np.inf
    with pytest.raises(ValueError):
        oracle.quantize(w)


# ---------------------------------------------------- double quantisation

def test_fixed_point_mean_is_the_mean_and_order_free():
    rng = np.random.default_rng(5)
    s = np.abs(rng.normal(0.05, 0.01, 5000)).astype(np.float32)
    mu = oracle.fixed_point_mean(s)
    exact = sum(Fraction(float(v)) for v in s) / len(s)
    assert abs(Fraction(float(mu)) - exact) <= exact * Fraction(1, 2 ** 22)
    for seed in range(3):
        perm = np.random.default_rng(seed).permutation(s)
        assert oracle.fixed_point_mean(perm) == mu
    assert oracle.fixed_point_mean(np.zeros(10, np.float32)) == 0.0
    assert oracle.fixed_point_mean(np.full(7, 0.375, np.float32)) == np.float32(0.375)


def test_double_quant_codes_are_nearest_int8_codes():
    rng = np.random.default_rng(6)
    s = np.abs(rng.normal(0.05, 0.012, 700)).astype(np.float32)
    q, f, mu = oracle.double_quantize(s, 256)
    assert f.size == 3 and q.dtype == np.int8
    assert np.all(np.abs(q.astype(int)) <= 127)
    c = (s - mu).astype(np.float32)
    for g in range(3):
        sl = slice(256 * g, min(256 * g + 256, 700))
        cg, qg = c[sl], q[sl]
        k = int(np.argmax(np.abs(cg)))
        assert abs(int(qg[k])) == 127 and np.sign(qg[k]) == np.sign(cg[k])
        fg = Fraction(float(f[g]))
        for cb, qb in zip(cg, qg):
            t = Fraction(float(cb)) / fg
            frac = t - (t.numerator // t.denominator)
            if abs(frac - Fraction(1, 2)) < Fraction(1, 10 ** 5):
                continue                                   # near a tie: rounding of c/f decides
            best = min(range(-127, 128), key=lambda v: abs(Fraction(float(cb)) - v * fg))
            assert int(qb) == best


def test_double_quant_reconstruction_error_bound():
    rng = np.random.default_rng(8)
    s = np.abs(rng.normal(0.05, 0.012, 3000)).astype(np.float32)
    q, f, mu = oracle.double_quantize(s, 256)
    sh = oracle.dequantize_scales(q, f, mu, 256)
    f_el = np.repeat(f, 256)[:s.size].astype(np.float64)
    err = np.abs(sh.astype(np.float64) - s.astype(np.float64))
    assert np.all(err <= 0.5 * f_el * (1 + 1e-5) + 4 * np.spacing(s).astype(np.float64))


def test_quantize_end_to_end_error_on_gaussian_weights():
    rng = np.random.default_rng(9)
    w = (rng.standard_normal(64 * 512) * 0.02).astype(np.float32)
    qt = oracle.quantize(w, 64, 256)
    w_hat = oracle.dequantize(qt)
    s_hat = np.repeat(oracle.block_scales(qt), 64)
    # nearest-level error (<= half the widest gap of the table) plus the scale error
    half_gap = float(np.max(np.diff(oracle.nf4_levels().astype(np.float64)))) / 2
    bound = half_gap * np.repeat(qt["absmax"], 64) + np.abs(s_hat - np.repeat(qt["absmax"], 64))
    assert np.all(np.abs(w_hat - w) <= bound * (1 + 1e-5) + 1e-9)
    rel = np.linalg.norm(w_hat - w) / np.linalg.norm(w)
    assert rel < 0.12


# ------------------------------------------------------------ storage cost

def test_storage_bits_match_the_pages(golden):
    g = golden("storage_bits.txt")
    n = 4096 * 11008
    dq = oracle.storage_bits(n, 64, 256)
    assert round(dq["bits_per_weight"], 2) == float(g["nf4_b64_dq256_bits_per_weight_approx"][0])
    assert abs(dq["bits_per_weight"] - (4 + 8 / 64 + 32 / (64 * 256))) < 1e-6
    toy = oracle.storage_bits(4, 4, 0)
    assert 8 * (toy["codes"] + toy["factors"]) == int(g["toy_group_of_4_fp32_scale_bits"][0])
    assert 4 * 16 == int(g["toy_group_of_4_fp16_bits"][0])
    b64 = oracle.storage_bits(64, 64, 0)
    assert 8 * (b64["codes"] + b64["factors"]) == int(g["block64_fp32_scale_bits"][0])
    assert b64["bits_per_weight"] == float(g["block64_fp32_scale_bits_per_weight"][0])
