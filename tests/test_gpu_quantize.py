"""GPU parity of quantise / double-quantise / dequantise against the oracle.

Bit-exact: packed indices, int8 scale codes, group factors, the mean, and
the fp32 dequantised weight; the bf16 dequantised weight is the fp32 one
rounded to nearest even.
"""

import numpy as np
import pytest
import torch

import oracle
from bit_nf4_quantized_17_b200 import qlora as Q
from bit_nf4_quantized_17_b200 import workloads as WL

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bits(a):
    return np.ascontiguousarray(a).view(np.uint32)


def _check(W_cpu, bs=64, dq=256, table=Q.QLORA_TABLE_NF4):
    levels = oracle.nf4_levels() if table == Q.QLORA_TABLE_NF4 else oracle.uniform_levels()
    ref = oracle.quantize(W_cpu.float().numpy(), bs, dq, levels)
    q = Q.qlora_quantize(W_cpu.to(DEV), bs, dq, table)
    assert np.array_equal(q.codes.cpu().numpy(), ref["codes"])
    if dq:
        nb = ref["scale_codes"].size
        assert np.array_equal(q.scale_codes.cpu().numpy()[:nb], ref["scale_codes"])
        assert np.array_equal(_bits(q.factors.cpu().numpy()), _bits(ref["factors"]))
        assert _bits(q.mean.cpu().numpy()[:1])[0] == _bits(np.array([ref["mean"]], np.float32))[0]
    else:
        assert np.array_equal(_bits(q.factors.cpu().numpy()), _bits(ref["factors"]))
    w_hat = oracle.dequantize(ref).reshape(W_cpu.shape)
    got32 = Q.qlora_dequantize(q, torch.float32).cpu().numpy()
    assert np.array_equal(_bits(got32), _bits(w_hat))
    got16 = Q.qlora_dequantize(q, torch.bfloat16).view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got16, oracle.f32_to_bf16_bits(w_hat))
    return q, ref


def test_single_linear_fp32_weights():
    shape = WL.WORKLOADS["single_256"].linears[0]
    _check(WL.weight(shape, 0))


def test_attention_projection_with_outliers():
    shape = WL.WORKLOADS["attn_4096"].linears[0]
    W = WL.weight(shape, 0)
    assert (W.float().abs() > 0.15).sum() > 1000     # the outliers are present
    _check(W)


@pytest.mark.parametrize("j", [0, 1])
def test_mlp_shapes(j):
    shape = WL.WORKLOADS["mlp_11008"].linears[j]
    _check(WL.weight(shape, 16 * j))


@pytest.mark.parametrize("rows,cols,bs,dq", [
    (3, 5, 64, 256),          # n = 15: one partial block, odd element count
    (1, 1, 64, 256),
    (17, 100, 64, 256),       # blocks straddle rows, partial last block
    (300, 64, 128, 64),
    (129, 512, 256, 1024),
    (64, 1024, 512, 256),
    (8, 4096, 1024, 256),
    (123, 77, 64, 0),         # no double quantisation: fp32 absmax stored
    (1024, 1024, 64, 1024),
])
def test_ragged_and_blocksize_variants(rows, cols, bs, dq):
    W = WL.randn((rows, cols), 0.02, 99 + rows, torch.float32)
    _check(W, bs, dq)


def test_uniform_table_and_worked_example():
    # the page's group of four, padded with zeros to one block of 64
    w = torch.zeros(1, 64, dtype=torch.float32)
    w[0, :4] = torch.tensor([0.27, 0.58, -0.75, 1.52])
    q, ref = _check(w, 64, 0, Q.QLORA_TABLE_UNIFORM)
    idx = oracle.unpack_nibbles(q.codes.cpu().numpy(), 64)
    assert list(idx[:4]) == [9, 10, 4, 15]
    assert abs(float(Q.qlora_dequantize(q)[0, 0]) - 0.304) < 1e-6
    W = WL.randn((64, 640), 0.02, 5, torch.bfloat16)
    _check(W, 64, 256, Q.QLORA_TABLE_UNIFORM)


def test_zero_blocks_and_constant_scale():
    W = torch.zeros(16, 256, dtype=torch.float32)
    W[8:] = WL.randn((8, 256), 1.0, 3, torch.float32)
    _check(W)
    # every block has the same absmax: mean = scale, codes and factors all zero
    lv = torch.tensor(oracle.nf4_levels())
    idx = torch.randint(0, 16, (64, 64), generator=torch.Generator().manual_seed(1))
    idx[:, 0] = 15
    W = (lv[idx] * 0.03125).float()
    q, ref = _check(W)
    assert torch.count_nonzero(q.factors) == 0
    assert torch.equal(Q.qlora_dequantize(q).cpu(), W)


def test_nonfinite_weight_is_reported():
    W = WL.randn((4, 128), 0.02, 1, torch.float32)
    W[2, 7] = float("nan")
    with pytest.raises(Q.QloraError) as e:
        Q.qlora_quantize(W.to(DEV))
    assert e.value.status == Q.QLORA_ERR_NONFINITE
    W[2, 7] = float("inf")
    with pytest.raises(Q.QloraError) as e:
        Q.qlora_quantize(W.to(DEV))
    assert e.value.status == Q.QLORA_ERR_NONFINITE


def _threshold_weights(levels, scales, blocks_per_scale, seed):
    """fp32 weights whose normalised values x = w / s sit on the decision
    thresholds of `levels` and on their -3..+3 fp32 neighbours.

    Every block of 64 holds one element +-s (so its absmax is exactly s) and
    63 values w = m s moved by -3..+3 ulps, m the exact midpoint of two
    adjacent levels (fp64; the decision boundary of the nearest-level rule).
    With s = 1 the normalised value is w itself, so the kernel's comparison
    meets each threshold and its neighbours exactly; other scales put
    RN(w / s) within a few ulps of the thresholds, where the library's cell
    lookup hands over to its IEEE-division fallback."""
    q = np.asarray(levels, np.float32).astype(np.float64)
    mids = (q[:-1] + q[1:]) * 0.5
    rng = np.random.default_rng(seed)
    blocks = []
    for s in scales:
        s32 = np.float32(s)
        vals = []
        for m in mids:
            c = np.float32(m * np.float64(s32))
            for d in range(-3, 4):
                v = c
                for _ in range(abs(d)):
                    v = np.nextafter(v, np.float32(np.inf if d > 0 else -np.inf), dtype=np.float32)
                vals.append(v)
        vals = np.array(vals, np.float32)
        assert np.all(np.abs(vals) < s32)
        for b in range(blocks_per_scale):
            pick = rng.permutation(np.resize(rng.permutation(vals), 63))
            block = np.concatenate([[s32 if b % 2 == 0 else -s32], pick]).astype(np.float32)
            blocks.append(rng.permutation(block))
    return np.stack(blocks).reshape(-1, 1024)


@pytest.mark.parametrize("table", [Q.QLORA_TABLE_NF4, Q.QLORA_TABLE_UNIFORM])
@pytest.mark.parametrize("dq", [256, 0])
def test_values_on_every_decision_threshold(table, dq):
    # codes must match the oracle bit for bit exactly where the nearest level
    # changes (ties take the lower index), for unit and non-unit scales
    levels = oracle.nf4_levels() if table == Q.QLORA_TABLE_NF4 else oracle.uniform_levels()
    scales = [1.0, 0.5, 2.0, 0.02, 0.0173, 3.7, 1e-3, 0.3, 7.25, 1.5 * 2.0 ** -126, 3e-39]
    W = torch.from_numpy(_threshold_weights(levels, scales, 32, 21 + table))
    _, ref = _check(W, 64, dq, table)
    # the inputs do reach every index on both sides of every threshold
    assert set(np.unique(ref["idx"]).tolist()) == set(range(16))
