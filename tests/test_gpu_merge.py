"""GPU parity of qlora_merge: the adapter merged into a restored bf16 weight.

W_merged = bf16(W_hat + (alpha/r) B A) with W_hat the fp32 dequantised
weight ("LoRA 与 QLoRA：把大模型微调拆成可负担的工程", section 3).  The library
accumulates the rank-r update in fp32 and rounds once to bf16: every element
is within one bf16 ulp of the oracle's exact sum rounded to bf16.  With B = 0
the result is the compute weight bf16(W_hat) bit for bit.  (That the merged
weight reproduces the layer's forward pass in exact arithmetic is pinned on
the oracle.)
"""

import numpy as np
import pytest
import torch

import oracle
from bit_nf4_quantized_17_b200 import qlora as Q
from bit_nf4_quantized_17_b200 import workloads as WL
from parity import assert_close, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bf16_bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16).astype(np.int32)


def _ulp_distance(gpu_bits, ref_f32):
    ref_bits = oracle.f32_to_bf16_bits(np.asarray(ref_f32, np.float32)).astype(np.uint16).astype(np.int32)
    # bf16 bit patterns of the same sign order like their values
    return np.abs(gpu_bits - ref_bits)


@pytest.mark.parametrize("bs,dq,table", [(64, 256, Q.QLORA_TABLE_NF4), (128, 0, Q.QLORA_TABLE_UNIFORM)])
def test_merge_matches_oracle(bs, dq, table):
    shape = WL.WORKLOADS["attn_4096"].linears[0]
    inp = WL.linear_inputs(shape, 8, 5)
    W, A, B, X = inp["W"], inp["A"], inp["B"], inp["X"]
    B = WL.randn(B.shape, 0.05, 9, torch.bfloat16)
    levels = oracle.uniform_levels() if table == Q.QLORA_TABLE_UNIFORM else oracle.nf4_levels()
    q = Q.qlora_quantize(W.to(DEV), blocksize=bs, dq_blocksize=dq, table=table)
    out = Q.qlora_merge(q, A.to(DEV), B.to(DEV), shape.alpha)
    torch.cuda.synchronize()
    ref = oracle.quantize(W.float().numpy(), bs, dq, levels=levels)
    w_hat = oracle.dequantize(ref).reshape(W.shape)
    exact = oracle.merge_weight(w_hat, A.float().numpy(), B.float().numpy(), shape.alpha)
    # Bound: one bf16 ulp of the exact value, plus the fp32 error of the sum
    # (r products, the scaling and the addition, each rounded: (r + 2) 2^-24
    # of the magnitudes summed), which dominates only where W_hat and the
    # update nearly cancel.
    r = A.shape[0]
    s = oracle.lora_scale(shape.alpha, r)
    mag = np.abs(w_hat.astype(np.float64)) + s * (np.abs(B.float().numpy()).astype(np.float64)
                                                  @ np.abs(A.float().numpy()).astype(np.float64))
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(exact), 1e-38))) - 7)
    err = np.abs(f64(out) - exact)
    assert np.all(err <= ulp + (r + 2) * 2.0 ** -24 * mag)
    # and nearly always the same bf16 as the exact value rounded once
    dist = _ulp_distance(_bf16_bits(out), exact.astype(np.float32))
    assert np.mean(dist == 0) > 0.99
    # used as a plain bf16 weight, it gives the product of the oracle's merged
    # weight rounded to bf16 (the merged layer's output, at the bf16 tolerance)
    merged_bf16 = oracle.round_to_bf16(exact.astype(np.float32)).astype(np.float64)
    assert_close(f64(X) @ f64(out).T, f64(X) @ merged_bf16.T, "X W_merged^T")


def test_merge_with_zero_b_is_the_compute_weight():
    W = WL.randn((192, 512), 0.02, 11, torch.bfloat16)
    A = WL.randn((8, 512), 0.35, 12, torch.bfloat16)
    q = Q.qlora_quantize(W.to(DEV))
    out = Q.qlora_merge(q, A.to(DEV), torch.zeros((192, 8), dtype=torch.bfloat16, device=DEV), 16.0)
    torch.cuda.synchronize()
    ref = oracle.compute_weight(oracle.quantize(W.float().numpy(), 64, 256)).reshape(192, 512)
    assert np.array_equal(out.float().cpu().numpy(), ref)


def _bound_ok(out, exact, base_abs, A, B, s, r):
    # one bf16 ulp of the exact value plus the fp32 error of the rank-r sum
    mag = base_abs + s * (np.abs(f64(B)) @ np.abs(f64(A)))
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(exact), 1e-38))) - 7)
    return np.all(np.abs(f64(out) - exact) <= ulp + (r + 2) * 2.0 ** -24 * mag)


def test_merge_dense_matches_oracle_and_works_in_place():
    W = WL.randn((320, 1024), 0.02, 21, torch.bfloat16)
    A = WL.randn((16, 1024), 0.25, 22, torch.bfloat16)
    B = WL.randn((320, 16), 0.05, 23, torch.bfloat16)
    Wd, Ad, Bd = W.to(DEV), A.to(DEV), B.to(DEV)
    out = Q.qlora_merge_dense(Wd, Ad, Bd, 32.0)
    inplace = Wd.clone()
    Q.qlora_merge_dense(inplace, Ad, Bd, 32.0, out=inplace)
    torch.cuda.synchronize()
    exact = oracle.merge_weight(f64(W), f64(A), f64(B), 32.0)
    assert _bound_ok(out, exact, np.abs(f64(W)), A, B, oracle.lora_scale(32.0, 16), 16)
    assert torch.equal(out, inplace)


def test_unmerge_restores_the_compute_weight():
    # merge then merge_dense with -alpha: back to bf16(W_hat) up to the two roundings
    W = WL.randn((256, 768), 0.02, 31, torch.bfloat16)
    A = WL.randn((8, 768), 0.35, 32, torch.bfloat16)
    B = WL.randn((256, 8), 0.05, 33, torch.bfloat16)
    q = Q.qlora_quantize(W.to(DEV))
    Ad, Bd = A.to(DEV), B.to(DEV)
    merged = Q.qlora_merge(q, Ad, Bd, 16.0)
    back = Q.qlora_merge_dense(merged, Ad, Bd, -16.0)
    torch.cuda.synchronize()
    # the unmerge step itself is the oracle's sum on the merged bf16 weight
    exact = oracle.merge_weight(f64(merged), f64(A), f64(B), -16.0)
    s = oracle.lora_scale(16.0, 8)
    assert _bound_ok(back, exact, np.abs(f64(merged)), A, B, s, 8)
    # and it lands next to the compute weight: within the two bf16 roundings
    w_bf16 = oracle.compute_weight(oracle.quantize(W.float().numpy(), 64, 256)).reshape(256, 768)
    upd = s * (np.abs(f64(B)) @ np.abs(f64(A)))
    tol = 2.0 ** -7 * (np.abs(w_bf16) + upd) + 1e-30
    assert np.all(np.abs(f64(back) - w_bf16) <= tol)


@pytest.mark.parametrize("N,K,r", [(200, 576, 40), (136, 320, 64), (64, 128, 1)])
def test_merge_ranks_over_chunks_and_ragged_tiles(N, K, r):
    # r = 40: one full 32-rank chunk and a partial one; r = 64: two full ones;
    # N and K leave partial 64-row and 128-column tiles
    W = WL.randn((N, K), 0.02, 41, torch.bfloat16)
    A = WL.randn((r, K), 0.3, 42, torch.bfloat16)
    B = WL.randn((N, r), 0.05, 43, torch.bfloat16)
    q = Q.qlora_quantize(W.to(DEV))
    out = Q.qlora_merge(q, A.to(DEV), B.to(DEV), 16.0)
    torch.cuda.synchronize()
    w_hat = oracle.dequantize(oracle.quantize(W.float().numpy(), 64, 256)).reshape(N, K)
    exact = oracle.merge_weight(w_hat, f64(A), f64(B), 16.0)
    assert _bound_ok(out, exact, np.abs(w_hat.astype(np.float64)), A, B, oracle.lora_scale(16.0, r), r)


@pytest.mark.parametrize("r", [136, 256])
def test_merge_ranks_over_several_stages(r):
    # r = 136: three 64-rank stages, the last with one 16-rank step; r = 256: four
    # full stages through a two-stage ring; both forms (NF4 base and dense base)
    N, K = 160, 320
    W = WL.randn((N, K), 0.02, 51, torch.bfloat16)
    A = WL.randn((r, K), 0.1, 52, torch.bfloat16)
    B = WL.randn((N, r), 0.05, 53, torch.bfloat16)
    Ad, Bd = A.to(DEV), B.to(DEV)
    q = Q.qlora_quantize(W.to(DEV))
    out = Q.qlora_merge(q, Ad, Bd, 32.0)
    dense = Q.qlora_merge_dense(W.to(DEV), Ad, Bd, 32.0)
    torch.cuda.synchronize()
    s = oracle.lora_scale(32.0, r)
    w_hat = oracle.dequantize(oracle.quantize(W.float().numpy(), 64, 256)).reshape(N, K)
    exact = oracle.merge_weight(w_hat, f64(A), f64(B), 32.0)
    assert _bound_ok(out, exact, np.abs(w_hat.astype(np.float64)), A, B, s, r)
    exact_d = oracle.merge_weight(f64(W), f64(A), f64(B), 32.0)
    assert _bound_ok(dense, exact_d, np.abs(f64(W)), A, B, s, r)
