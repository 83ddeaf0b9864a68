"""qlora_quantize_noalloc: quantisation for callers that cannot allocate a
workspace (device memory owned by a pool that already reserved the GPU, or
loops that cannot pay cudaMalloc's device-wide synchronisation).

Its results must equal qlora_quantize's bit for bit (the tolerance of every
quantisation test), on two calls in a row: the fixed device array it uses in
place of a workspace keeps the previous call's contents, so the second call
checks that nothing leaks from the first.  This file is collected last so that
a run stopping at the first failure has already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

from bit_nf4_quantized_17_b200 import qlora as Q
from bit_nf4_quantized_17_b200 import workloads as WL

pytestmark = pytest.mark.gpu


def _noalloc_fn():
    fn = Q.lib().qlora_quantize_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.POINTER(Q.qlora_nf4),
                   ctypes.c_void_p, ctypes.c_void_p]
    return fn


def _quantize_noalloc(W, blocksize, dq_blocksize, table=Q.QLORA_TABLE_NF4):
    q = Q.QuantizedWeight.empty(W.shape[0], W.shape[1], blocksize, dq_blocksize, table,
                                W.device)
    status = torch.full((1,), 12345, dtype=torch.int32, device=W.device)
    st = q.struct
    dtype = Q.QLORA_BF16 if W.dtype == torch.bfloat16 else Q.QLORA_F32
    rc = _noalloc_fn()(ctypes.c_void_p(W.data_ptr()), dtype, ctypes.byref(st),
                       ctypes.c_void_p(status.data_ptr()), Q._stream())
    assert rc == Q.QLORA_OK, Q.qlora_status_string(rc)
    torch.cuda.synchronize()
    return q, int(status.item())


def _same(a, b):
    # without double quantisation scale_codes and mean are unused placeholders
    names = ("codes", "scale_codes", "factors", "mean") if a.dq_blocksize else ("codes", "factors")
    for name in names:
        x = getattr(a, name).cpu().numpy()
        y = getattr(b, name).cpu().numpy()
        assert np.array_equal(x.view(np.uint8), y.view(np.uint8)), name


def test_noalloc_quantize_matches_workspace_quantize_twice_in_a_row():
    dev = torch.device("cuda")
    cases = [
        (WL.weight(WL.WORKLOADS["attn_4096"].linears[0], 0, dev), 64, 256),
        (WL.randn((1000, 640), 0.02, 77, torch.float32, dev), 128, 64),
    ]
    for W, bs, dq in cases:
        got, status = _quantize_noalloc(W, bs, dq)
        ref = Q.qlora_quantize(W, bs, dq)
        assert status == 0
        _same(got, ref)


def test_noalloc_quantize_refuses_tensors_beyond_its_array():
    # 2^20 blocks of 64 fit; one more block does not.  Refused before any GPU work.
    big = Q.qlora_nf4(1 << 20, 65, 64, 256, 0, 0, 0x10000, 0x20000, 0x30000, 0x40000)
    rc = _noalloc_fn()(ctypes.c_void_p(0x50000), Q.QLORA_BF16, ctypes.byref(big), None, None)
    assert rc == Q.QLORA_ERR_WORKSPACE


def test_noalloc_quantize_at_the_array_limit_and_without_double_quant():
    # exactly 2^20 blocks with double quantisation is accepted; without it
    # only the header of the array is used, so a larger tensor is accepted too
    dev = torch.device("cuda")
    W = WL.randn((1024, 65536), 0.02, 91, torch.bfloat16, dev)        # 2^20 blocks of 64
    got, status = _quantize_noalloc(W, 64, 256)
    assert status == 0
    _same(got, Q.qlora_quantize(W, 64, 256))
    W2 = WL.randn((1025, 65536), 0.02, 92, torch.bfloat16, dev)       # 2^20 + 1024 blocks
    for table in (Q.QLORA_TABLE_NF4, Q.QLORA_TABLE_UNIFORM):
        got, status = _quantize_noalloc(W2, 64, 0, table)
        assert status == 0
        _same(got, Q.qlora_quantize(W2, 64, 0, table))


def test_noalloc_nonfinite_status_does_not_carry_over():
    # a NaN weight reports QLORA_ERR_NONFINITE through status_out; the next
    # call on a clean weight reports 0 and equals qlora_quantize bit for bit
    dev = torch.device("cuda")
    W = WL.randn((512, 1024), 0.02, 93, torch.float32, dev)
    bad = W.clone()
    bad[17, 300] = float("nan")
    _, status = _quantize_noalloc(bad, 64, 256)
    assert status == Q.QLORA_ERR_NONFINITE
    got, status = _quantize_noalloc(W, 64, 256)
    assert status == 0
    _same(got, Q.qlora_quantize(W, 64, 256))
