"""Failure detection on the GPU, without faulting it, and output bounds.

- A bounded wait that runs out (on an mbarrier nothing completes) surfaces as
  QLORA_ERR_DEVICE_TIMEOUT through the workspace status word; qlora_check
  clears it and the context stays usable for the next calls.
- Guard bands around every output buffer stay untouched: the kernels write
  exactly their outputs, on ragged shapes of every path.
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


def test_bounded_wait_reports_timeout_and_the_context_survives():
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    Q.qlora_selftest_timeout(2_000_000, ws)  # about a millisecond
    with pytest.raises(Q.QloraError) as e:
        Q.qlora_check(ws)
    assert e.value.status == Q.QLORA_ERR_DEVICE_TIMEOUT
    Q.qlora_check(ws)  # cleared
    # the context still runs the layer correctly
    shape = WL.WORKLOADS["single_256"].linears[0]
    inp = WL.linear_inputs(shape, 16, 0)
    q = Q.qlora_quantize(inp["W"].to(DEV))
    Y = Q.qlora_linear_fwd(q, inp["A"].to(DEV), inp["B"].to(DEV), shape.alpha, inp["X"].to(DEV),
                           check=True)
    w_hat = oracle.compute_weight(oracle.quantize(inp["W"].numpy(), 64, 256)).reshape(256, 256)
    y_ref, _ = oracle.linear_fwd(w_hat, f64(inp["A"]), f64(inp["B"]), shape.alpha, f64(inp["X"]))
    assert_close(f64(Y), y_ref, "Y")


GUARD = 4096  # elements before and after each output


def _guarded(shape, dtype):
    n = int(np.prod(shape))
    buf = torch.empty(n + 2 * GUARD, dtype=dtype, device=DEV)
    buf.view(torch.uint8).fill_(0xA5)
    return buf, buf[GUARD:GUARD + n].view(*shape)


def _guards_intact(buf):
    raw = buf.view(torch.uint8).cpu().numpy()
    es = buf.element_size()
    return bool((raw[:GUARD * es] == 0xA5).all() and (raw[-GUARD * es:] == 0xA5).all())


@pytest.mark.parametrize("M,N,K,r", [(1, 1032, 1024, 16), (13, 520, 2048, 24), (700, 776, 640, 16),
                                     (1500, 2600, 1024, 16)])
def test_outputs_stay_inside_their_buffers(M, N, K, r):
    shape = WL.LinearShape(N, K, r, 2.0 * r)
    inp = WL.linear_inputs(shape, M, 40 + M)
    q = Q.qlora_quantize(inp["W"].to(DEV))
    A, B, X, dY = (inp[k].to(DEV) for k in ("A", "B", "X", "dY"))
    bufs = {}
    bufs["Y"], Y = _guarded((M, N), torch.bfloat16)
    bufs["U"], U = _guarded((M, r), torch.float32)
    bufs["dX"], dX = _guarded((M, K), torch.bfloat16)
    bufs["dA"], dA = _guarded((r, K), torch.float32)
    bufs["dB"], dB = _guarded((N, r), torch.float32)
    Q.qlora_linear_fwd(q, A, B, shape.alpha, X, Y=Y, U_save=U, check=True)
    Q.qlora_linear_bwd(q, A, B, shape.alpha, X, U, dY, dX=dX, dA=dA, dB=dB, check=True)
    torch.cuda.synchronize()
    for name, buf in bufs.items():
        assert _guards_intact(buf), f"{name}: a guard band was written"
    w_hat = oracle.compute_weight(oracle.quantize(inp["W"].float().numpy(), 64, 256)).reshape(N, K)
    rows = slice(None) if M <= 64 else np.arange(0, M, max(1, M // 40))
    y_ref, _ = oracle.linear_fwd(w_hat, f64(inp["A"]), f64(inp["B"]), shape.alpha, f64(inp["X"])[rows])
    assert_close(f64(Y)[rows], y_ref, "Y")
