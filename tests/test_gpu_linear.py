"""GPU parity of the QLoRA linear forward and backward against the oracle.

Forward Y = X W^T + s (X A^T) B^T and backward dX = dY W + s V A,
dB = s dY^T U, dA = s V^T X (V = dY B), with W the oracle's own dequantised
weight rounded to bf16 (the compute dtype the pages name).  bf16 outputs
within the stated tolerance (tests/parity.py); fp32 U, dA, dB within the same
bar measured in their own scale.  At the full sizes the oracle checks
sampled token rows of Y and dX and every element of U, dA and dB.
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


def _w_hat(W_cpu):
    ref = oracle.quantize(W_cpu.float().numpy(), 64, 256)
    return oracle.compute_weight(ref).reshape(W_cpu.shape)


def _run(inp, alpha, rows=None, w_hat=None, check=True):
    """Run fwd + bwd on the GPU and compare with the oracle (optionally on a
    subset of token rows for Y and dX)."""
    W, A, B, X, dY = (inp[k] for k in ("W", "A", "B", "X", "dY"))
    M, r = X.shape[0], A.shape[0]
    q = Q.qlora_quantize(W.to(DEV))
    Ad, Bd, Xd, dYd = (t.to(DEV) for t in (A, B, X, dY))
    U = torch.empty((M, r), dtype=torch.float32, device=DEV)
    Y = Q.qlora_linear_fwd(q, Ad, Bd, alpha, Xd, U_save=U, check=True)
    dX, dA, dB = Q.qlora_linear_bwd(q, Ad, Bd, alpha, Xd, U, dYd, check=True)
    torch.cuda.synchronize()
    if not check:
        return q, Y, U, dX, dA, dB
    w_hat = _w_hat(W) if w_hat is None else w_hat
    a, b, x, dy = f64(A), f64(B), f64(X), f64(dY)
    sel = slice(None) if rows is None else rows
    y_ref, _ = oracle.linear_fwd(w_hat, a, b, alpha, x[sel])
    assert_close(f64(Y)[sel], y_ref, "Y")
    u_ref = oracle.lora_down(a, x)
    assert_close_scaled(U, u_ref, "U")
    dx_ref, _, _ = oracle.linear_bwd(w_hat, a, b, alpha, x[sel], dy[sel])
    assert_close(f64(dX)[sel], dx_ref, "dX")
    da_ref, db_ref = oracle.lora_grads(a, b, alpha, x, dy)
    assert_close_scaled(dA, da_ref, "dA")
    assert_close_scaled(dB, db_ref, "dB")
    return q, Y, U, dX, dA, dB


def _inputs(d_out, d_in, r, M, seed, w_std=0.02, b_std=0.01):
    shape = WL.LinearShape(d_out, d_in, r, 2.0 * r, w_std=w_std)
    inp = WL.linear_inputs(shape, M, seed)
    if b_std != 0.01:
        inp["B"] = WL.randn((d_out, r), b_std, seed + 2, torch.bfloat16)
    return inp, shape.alpha


def test_single_linear_256():
    shape = WL.WORKLOADS["single_256"].linears[0]
    _run(WL.linear_inputs(shape, 16, 0), shape.alpha)


@pytest.mark.parametrize("M,N,K,r", [
    (1, 64, 64, 1), (3, 80, 192, 5), (17, 200, 128, 16), (130, 96, 320, 64),
    (257, 384, 256, 8), (64, 128, 4096, 256), (300, 1000, 640, 24),
    # more output tiles than SMs, ragged edges (CTA-pair kernels)
    (4000, 2600, 640, 16), (4000, 640, 2624, 16),
    # two tokens (dequant GEMVs): K below one 1024-column group, and a ragged second group
    (2, 200, 320, 16), (2, 4104, 1088, 24),
    # ranks that need more LoRA stages than the pipeline has slots: CTA pairs,
    # decode sizes, and a rank that is not a multiple of 64
    (600, 512, 1024, 256), (520, 384, 704, 200), (1, 1024, 1024, 256), (16, 520, 2048, 136),
])
def test_ragged_shapes(M, N, K, r):
    inp, alpha = _inputs(N, K, r, M, 1000 + M, b_std=0.05)
    _run(inp, alpha)


@pytest.fixture(scope="module")
def attn():
    shape = WL.WORKLOADS["attn_4096"].linears[0]
    inp = WL.linear_inputs(shape, 4096, 0)
    return shape, inp, _w_hat(inp["W"])


def test_attention_projection_4096(attn):
    shape, inp, w_hat = attn
    rows = np.sort(np.random.default_rng(0).choice(4096, 96, replace=False))
    rows = np.concatenate([[0], rows, [4095]])
    q, Y, U, dX, dA, dB = _run(inp, shape.alpha, rows=rows, w_hat=w_hat)
    # the same call again gives the same bits (fixed split points and summation order)
    A, B, X, dY = (inp[k].to(DEV) for k in ("A", "B", "X", "dY"))
    Y2 = Q.qlora_linear_fwd(q, A, B, shape.alpha, X)
    dX2, dA2, dB2 = Q.qlora_linear_bwd(q, A, B, shape.alpha, X, U, dY)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y2) and torch.equal(dX, dX2)
    assert torch.equal(dA, dA2) and torch.equal(dB, dB2)


@pytest.mark.parametrize("M", [5120, 7168])
def test_rank_splits_that_do_not_divide_the_row_tile(attn, M):
    """5120 and 7168 tokens split the contraction of U = X A^T and V = dY B
    7 and 5 ways when the clusters are resident (fewer otherwise): the
    cluster's reduce then gives its last CTA a shorter slice of the 128 rows."""
    shape, inp0, w_hat = attn
    inp = WL.linear_inputs(shape, M, 0)
    assert torch.equal(inp["W"], inp0["W"])  # the same W, so the same oracle weight
    rows = np.sort(np.random.default_rng(M).choice(M, 64, replace=False))
    rows = np.concatenate([[0], rows, [M - 1]])
    _run(inp, shape.alpha, rows=rows, w_hat=w_hat)


@pytest.fixture(scope="module", params=[0, 1], ids=["gate_up", "down"])
def mlp(request):
    shape = WL.WORKLOADS["mlp_11008"].linears[request.param]
    W = WL.weight(shape, 16 * request.param)
    return shape, request.param, W, _w_hat(W)


@pytest.mark.parametrize("M", [1, 16, 8192])
def test_mlp_shapes(mlp, M):
    shape, j, W, w_hat = mlp
    seed = 16 * j
    inp = dict(W=W, A=WL.lora_a(shape, seed), B=WL.lora_b(shape, seed),
               X=WL.activations(shape, M, seed), dY=WL.grad_output(shape, M, seed))
    rows = None
    if M > 64:
        rows = np.sort(np.random.default_rng(M).choice(M, 64, replace=False))
        rows = np.concatenate([[0], rows, [M - 1]])
    _run(inp, shape.alpha, rows=rows, w_hat=w_hat)


def _stack_linear(workload, j, layer, n_rows=32):
    """Linear j of layer `layer` of a stack workload at its token count, its
    seeds as the stack draws them; Y and dX checked on sampled token rows."""
    wl = WL.WORKLOADS[workload]
    shape, M = wl.linears[j], wl.tokens[0]
    inp = WL.linear_inputs(shape, M, WL.stack_seed(layer, j))
    rows = np.sort(np.random.default_rng(7 * layer + j).choice(M, n_rows, replace=False))
    rows = np.concatenate([[0], rows, [M - 1]])
    _run(inp, shape.alpha, rows=rows)


@pytest.mark.parametrize("j", range(7), ids=[n for n, _, _ in WL.LLAMA7B_LINEARS])
def test_stack_7b_layer_linears(j):
    # first and last layer of the 32-layer stack (different seeds)
    _stack_linear("stack_7b", j, 0)
    _stack_linear("stack_7b", j, 31, n_rows=8)


@pytest.mark.parametrize("j", [0, 4, 6], ids=["q_8192", "gate_22016x8192", "down_8192x22016"])
def test_stack_65b_linear_shapes(j):
    _stack_linear("stack_65b", j, 0)


def test_weight_with_zero_double_quant_factors():
    # every block has the same absmax: each group's centred scales are all 0,
    # so its factor is 0 and every block dequantises with the mean
    lv = torch.tensor(oracle.nf4_levels())
    idx = torch.randint(0, 16, (192, 512), generator=torch.Generator().manual_seed(3))
    idx[:, ::64] = 15
    inp, alpha = _inputs(192, 512, 16, 40, 21, b_std=0.05)
    inp["W"] = (lv[idx] * 0.03125).to(torch.bfloat16)
    q, *_ = _run(inp, alpha)
    assert torch.count_nonzero(q.factors) == 0
    inp1 = dict(inp)
    inp1["X"], inp1["dY"] = inp["X"][:1].clone(), inp["dY"][:1].clone()
    _run(inp1, alpha)


def test_zero_b_gives_base_output():
    inp, alpha = _inputs(192, 256, 8, 33, 7)
    inp["B"] = torch.zeros_like(inp["B"])
    q, Y, U, dX, dA, dB = _run(inp, alpha)
    base = f64(inp["X"]) @ _w_hat(inp["W"]).astype(np.float64).T
    assert_close(Y, base, "Y(B=0)")
    assert torch.count_nonzero(dA) == 0


def test_accumulate_recompute_skip_and_determinism():
    inp, alpha = _inputs(320, 384, 16, 70, 11, b_std=0.05)
    q, Y, U, dX, dA, dB = _run(inp, alpha)
    A, B, X, dY = (inp[k].to(DEV) for k in ("A", "B", "X", "dY"))
    # same inputs again: bit-identical outputs
    Y2 = Q.qlora_linear_fwd(q, A, B, alpha, X)
    assert torch.equal(Y, Y2)
    # U recomputed inside the backward when not given
    dX2, dA2, dB2 = Q.qlora_linear_bwd(q, A, B, alpha, X, None, dY)
    assert torch.equal(dX, dX2) and torch.equal(dA, dA2) and torch.equal(dB, dB2)
    # accumulate adds onto the given gradients
    dA3, dB3 = dA.clone(), dB.clone()
    Q.qlora_linear_bwd(q, A, B, alpha, X, U, dY, dA=dA3, dB=dB3, accumulate=True)
    torch.cuda.synchronize()
    assert torch.equal(dA3, dA + dA) and torch.equal(dB3, dB + dB)
    # dX may be skipped
    _, dA4, dB4 = Q.qlora_linear_bwd(q, A, B, alpha, X, U, dY, want_dx=False)
    assert torch.equal(dA4, dA) and torch.equal(dB4, dB)


def test_zero_tokens():
    inp, alpha = _inputs(128, 128, 8, 1, 3)
    q = Q.qlora_quantize(inp["W"].to(DEV))
    A, B = inp["A"].to(DEV), inp["B"].to(DEV)
    X = torch.empty((0, 128), dtype=torch.bfloat16, device=DEV)
    Y = Q.qlora_linear_fwd(q, A, B, alpha, X)
    assert Y.shape == (0, 128)
    dA = torch.full((8, 128), 5.0, device=DEV)
    dB = torch.full((128, 8), 5.0, device=DEV)
    Q.qlora_linear_bwd(q, A, B, alpha, X, None, torch.empty((0, 128), dtype=torch.bfloat16,
                                                            device=DEV), dA=dA, dB=dB)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dA) == 0 and torch.count_nonzero(dB) == 0


@pytest.mark.parametrize("M", [1, 2, 16, 700, 4096])
def test_cuda_graph_replay_matches_eager(M):
    # forward and backward captured in CUDA graphs (the backward forks onto a
    # second stream and joins back inside the graph) give the eager results
    # bit for bit, replay after replay
    shape = WL.LinearShape(1024, 2048, 16, 32.0)
    inp = WL.linear_inputs(shape, M, 900 + M)
    q = Q.qlora_quantize(inp["W"].to(DEV))
    A, B, X, dY = (inp[k].to(DEV) for k in ("A", "B", "X", "dY"))
    fb, bb = Q.qlora_linear_workspace(M, shape.d_out, shape.d_in, shape.r)
    fws = torch.zeros(fb, dtype=torch.uint8, device=DEV)
    bws = torch.zeros(bb, dtype=torch.uint8, device=DEV)
    Y = torch.empty((M, shape.d_out), dtype=torch.bfloat16, device=DEV)
    U = torch.empty((M, shape.r), dtype=torch.float32, device=DEV)
    dX = torch.empty((M, shape.d_in), dtype=torch.bfloat16, device=DEV)
    dA = torch.empty((shape.r, shape.d_in), dtype=torch.float32, device=DEV)
    dB = torch.empty((shape.d_out, shape.r), dtype=torch.float32, device=DEV)

    def step():
        Q.qlora_linear_fwd(q, A, B, shape.alpha, X, Y=Y, U_save=U, workspace=fws)
        Q.qlora_linear_bwd(q, A, B, shape.alpha, X, U, dY, dX=dX, dA=dA, dB=dB, workspace=bws)

    step()
    torch.cuda.synchronize()
    ref = [t.clone() for t in (Y, U, dX, dA, dB)]
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        with torch.cuda.graph(g, stream=cap):
            step()
    torch.cuda.current_stream().wait_stream(cap)
    for t in (Y, U, dX, dA, dB):
        t.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    for a, b in zip((Y, U, dX, dA, dB), ref):
        assert torch.equal(a, b)
    Q.qlora_check(fws)
    Q.qlora_check(bws)
    del g
