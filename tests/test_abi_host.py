"""Host-side checks of libqlora.so: it loads, exports every declared entry
point, and rejects bad arguments before touching the GPU (no CUDA call is
made by any test here)."""

import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from bit_nf4_quantized_17_b200 import qlora as Q

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for fname in os.listdir(os.path.join(ROOT, "include")):
        if not fname.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", fname), encoding="utf-8").read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(qlora_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    lib = Q.lib()
    names = _declared_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n


@pytest.mark.parametrize("table,ref", [(Q.QLORA_TABLE_NF4, oracle.nf4_levels),
                                       (Q.QLORA_TABLE_UNIFORM, oracle.uniform_levels)])
def test_library_level_table_matches_oracle_bits(table, ref):
    got = np.array(Q.qlora_levels(table), dtype=np.float32)
    assert np.array_equal(got.view(np.uint32), ref().view(np.uint32))


@pytest.mark.parametrize("rows,cols,bs,dq", [(4096, 11008, 64, 256), (256, 256, 64, 256),
                                             (7, 9, 64, 256), (1000, 1000, 128, 0),
                                             (33, 64, 1024, 1024)])
def test_sizes_match_oracle_storage(rows, cols, bs, dq):
    s = Q.qlora_nf4_sizes(rows, cols, bs, dq)
    o = oracle.storage_bits(rows * cols, bs, dq)
    assert s["codes"] == o["codes"]
    assert s["scale_codes"] == o["scale_codes"]
    assert s["factors"] == o["factors"]
    assert s["mean"] == o["mean"]


def test_size_query_rejects_bad_requests():
    with pytest.raises(Q.QloraError) as e:
        Q.qlora_nf4_sizes(0, 10)
    assert e.value.status == Q.QLORA_ERR_SHAPE
    for bs, dq in ((32, 256), (96, 256), (64, 100), (2048, 256)):
        with pytest.raises(Q.QloraError) as e:
            Q.qlora_nf4_sizes(64, 64, bs, dq)
        assert e.value.status == Q.QLORA_ERR_UNSUPPORTED
    with pytest.raises(Q.QloraError) as e:
        Q.qlora_nf4_sizes(1 << 20, 1 << 20)
    assert e.value.status == Q.QLORA_ERR_SHAPE


def _fake_q(rows=64, cols=128, bs=64, dq=256, base=0x10000):
    return Q.qlora_nf4(rows, cols, bs, dq, 0, 0, base, base + 0x1000, base + 0x2000, base + 0x3000)


def _call_quantize(q, w=0x40000, dtype=Q.QLORA_BF16, ws=0x80000, ws_bytes=1 << 20):
    return Q.lib().qlora_quantize(ctypes.c_void_p(w), dtype, ctypes.byref(q),
                                  ctypes.c_void_p(ws), ws_bytes, None)


def test_quantize_argument_errors():
    L = Q.lib()
    assert _call_quantize(_fake_q(), w=0) == Q.QLORA_ERR_NULL
    assert _call_quantize(_fake_q(), ws=0) == Q.QLORA_ERR_NULL
    assert L.qlora_quantize(ctypes.c_void_p(0x40000), 1, None, ctypes.c_void_p(0x80000), 1 << 20,
                            None) == Q.QLORA_ERR_NULL
    q = _fake_q()
    q.codes = None
    assert _call_quantize(q) == Q.QLORA_ERR_NULL
    q = _fake_q()
    q.mean = None
    assert _call_quantize(q) == Q.QLORA_ERR_NULL
    assert _call_quantize(_fake_q(), w=0x40001) == Q.QLORA_ERR_ALIGN
    assert _call_quantize(_fake_q(base=0x10008)) == Q.QLORA_ERR_ALIGN
    assert _call_quantize(_fake_q(bs=48)) == Q.QLORA_ERR_UNSUPPORTED
    assert _call_quantize(_fake_q(), dtype=7) == Q.QLORA_ERR_UNSUPPORTED
    assert _call_quantize(_fake_q(rows=0)) == Q.QLORA_ERR_SHAPE
    assert _call_quantize(_fake_q(), ws_bytes=100) == Q.QLORA_ERR_WORKSPACE
    q = _fake_q()
    q.table = 5
    assert _call_quantize(q) == Q.QLORA_ERR_UNSUPPORTED


def _call_fwd(q, r=8, M=16, A=0x100000, X=0x200000, Y=0x300000, ws=0x400000, ws_bytes=1 << 30):
    return Q.lib().qlora_linear_fwd(ctypes.byref(q), ctypes.c_void_p(A), ctypes.c_void_p(0x110000),
                                    r, 16.0, ctypes.c_void_p(X), M, ctypes.c_void_p(Y), None,
                                    ctypes.c_void_p(ws), ws_bytes, None)


def test_linear_argument_errors():
    q = _fake_q(256, 256)
    assert _call_fwd(q, A=0) == Q.QLORA_ERR_NULL
    assert _call_fwd(q, Y=0) == Q.QLORA_ERR_NULL
    assert _call_fwd(q, X=0x200004) == Q.QLORA_ERR_ALIGN
    assert _call_fwd(q, r=0) == Q.QLORA_ERR_SHAPE
    assert _call_fwd(q, r=257) == Q.QLORA_ERR_SHAPE
    assert _call_fwd(q, M=-1) == Q.QLORA_ERR_SHAPE
    assert _call_fwd(_fake_q(256, 200)) == Q.QLORA_ERR_UNSUPPORTED   # d_in % 64 != 0
    # blocks must not straddle rows: d_in a multiple of the block size
    assert _call_fwd(_fake_q(256, 384, bs=256)) == Q.QLORA_ERR_UNSUPPORTED
    assert _call_fwd(q, ws_bytes=16) == Q.QLORA_ERR_WORKSPACE
    # M = 0 passes validation and launches nothing
    assert _call_fwd(q, M=0) == Q.QLORA_OK
    L = Q.lib()
    rc = L.qlora_linear_bwd(ctypes.byref(q), ctypes.c_void_p(0x100000), ctypes.c_void_p(0x110000),
                            8, 16.0, ctypes.c_void_p(0x200000), None, None, 16, None,
                            ctypes.c_void_p(0x500000), ctypes.c_void_p(0x600000), 0,
                            ctypes.c_void_p(0x400000), 1 << 30, None)
    assert rc == Q.QLORA_ERR_NULL   # dY missing


def test_workspace_query_grows_with_problem():
    f1, b1 = Q.qlora_linear_workspace(16, 256, 256, 8)
    f2, b2 = Q.qlora_linear_workspace(4096, 4096, 4096, 16)
    assert 256 <= f1 < f2 and 256 <= b1 < b2
    with pytest.raises(Q.QloraError):
        Q.qlora_linear_workspace(16, 256, 256, 0)


def test_status_strings():
    for s in range(9):
        assert Q.qlora_status_string(s)
    assert Q.qlora_status_string(99) == "unknown status"


def test_timing_hook_rejects_bad_requests_without_cuda():
    L = Q.lib()
    # out-of-range launch budgets are refused before any event is created
    assert L.qlora_timing_begin(0x3, 0) == Q.QLORA_ERR_SHAPE
    assert L.qlora_timing_begin(0x3, 65537) == Q.QLORA_ERR_SHAPE
    # ending while timing is off
    assert L.qlora_timing_end(None, None) == Q.QLORA_ERR_UNSUPPORTED


def test_adamw_and_paged_argument_errors_without_cuda():
    L = Q.lib()
    P = ctypes.c_void_p
    a, b = P(0x20000), P(0x30000)

    def adamw(p=a, p16=None, g=b, m=a, v=b, n=8, step=1, lr=1e-3, b1=0.9, b2=0.999, eps=1e-8):
        return L.qlora_adamw(p, p16, g, m, v, n, step, lr, b1, b2, eps, 0.0, 1.0, None)

    assert adamw(n=0) == Q.QLORA_OK          # nothing to do: returns before any launch
    assert adamw(n=-1) == Q.QLORA_ERR_SHAPE
    assert adamw(step=0) == Q.QLORA_ERR_SHAPE
    assert adamw(g=None) == Q.QLORA_ERR_NULL
    assert adamw(m=P(0x20004)) == Q.QLORA_ERR_ALIGN
    assert adamw(p16=P(0x40002)) == Q.QLORA_ERR_ALIGN
    assert adamw(b2=1.0) == Q.QLORA_ERR_UNSUPPORTED
    assert adamw(b1=-0.1) == Q.QLORA_ERR_UNSUPPORTED
    assert adamw(eps=0.0) == Q.QLORA_ERR_UNSUPPORTED
    assert adamw(lr=float("nan")) == Q.QLORA_ERR_UNSUPPORTED
    out = P(1)
    assert L.qlora_paged_alloc(0, ctypes.byref(out)) == Q.QLORA_ERR_SHAPE and out.value is None
    assert L.qlora_paged_alloc(64, None) == Q.QLORA_ERR_NULL
    assert L.qlora_paged_prefetch(None, 64, 1, None) == Q.QLORA_ERR_NULL
    assert L.qlora_paged_prefetch(a, 0, 1, None) == Q.QLORA_ERR_SHAPE
    assert L.qlora_paged_free(None) == Q.QLORA_OK


def test_multi_adapter_argument_errors_without_cuda():
    L = Q.lib()
    q = _fake_q(256, 256)
    P = ctypes.c_void_p
    ws = Q.qlora_linear_workspace(4, 256, 256, 32)[0]

    def fwd(n=4, r=8, ids=P(0x50000), M=4):
        return L.qlora_linear_fwd_multi(ctypes.byref(q), P(0x100000), P(0x110000), n, r, 8.0, ids,
                                        P(0x120000), M, P(0x130000), None, P(0x140000), ws, None)

    assert fwd(n=0) == Q.QLORA_ERR_SHAPE
    assert fwd(n=33) == Q.QLORA_ERR_SHAPE          # 264 stacked ranks
    assert fwd(ids=None) == Q.QLORA_ERR_NULL
    assert fwd(ids=P(0x50002)) == Q.QLORA_ERR_ALIGN
    assert fwd(n=3, r=5) == Q.QLORA_ERR_UNSUPPORTED  # 15 stacked ranks
    assert fwd(M=0, ids=None) == Q.QLORA_OK          # nothing to do: no launch


def test_merge_dense_argument_errors_without_cuda():
    L = Q.lib()
    P = ctypes.c_void_p
    w, a, b, o = P(0x20000), P(0x30000), P(0x40000), P(0x50000)
    assert L.qlora_merge_dense(None, 8, 64, a, b, 8, 16.0, o, None) == Q.QLORA_ERR_NULL
    assert L.qlora_merge_dense(w, 8, 60, a, b, 8, 16.0, o, None) == Q.QLORA_ERR_SHAPE   # cols % 8
    assert L.qlora_merge_dense(w, 0, 64, a, b, 8, 16.0, o, None) == Q.QLORA_ERR_SHAPE
    assert L.qlora_merge_dense(w, 8, 64, a, b, 257, 16.0, o, None) == Q.QLORA_ERR_SHAPE
    assert L.qlora_merge_dense(w, 8, 64, P(0x30008), b, 8, 16.0, o, None) == Q.QLORA_ERR_ALIGN


def test_timeout_selftest_argument_errors_without_cuda():
    L = Q.lib()
    P = ctypes.c_void_p
    assert L.qlora_selftest_timeout(1000, None, None) == Q.QLORA_ERR_NULL
    assert L.qlora_selftest_timeout(0, P(0x10000), None) == Q.QLORA_ERR_SHAPE
    assert L.qlora_selftest_timeout(2 ** 33, P(0x10000), None) == Q.QLORA_ERR_SHAPE
    assert L.qlora_selftest_timeout(1000, P(0x10004), None) == Q.QLORA_ERR_ALIGN


def test_binding_checks_tensors_before_calling_the_library():
    # the library sees only pointers: a wrong shape, dtype or device raises in Python
    import torch
    from types import SimpleNamespace

    q = SimpleNamespace(rows=64, cols=128)
    A = torch.zeros(8, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="A"):
        Q._check_linear(q, 4, 16, A=A)                       # 8 rows for rank 16
    with pytest.raises(ValueError, match="keep_mask"):
        Q._check_linear(q, 4, 8, keep_mask=torch.zeros(4, 8, dtype=torch.uint8))  # K/8 = 16
    with pytest.raises(ValueError, match="adapter"):
        Q._check_linear(q, 4, 8, adapter=torch.zeros(4, dtype=torch.int64))
    with pytest.raises(ValueError, match="cpu"):
        Q._check_linear(q, 4, 8, A=A)                        # right shape, host memory


def test_quantize_binding_refuses_a_mismatched_output():
    # out's dimensions, not W's, would size the library's reads: they must agree
    import torch

    class FakeW:  # passes the binding's first checks without a GPU
        is_cuda = True
        shape = (64, 128)
        dtype = torch.bfloat16

        def dim(self):
            return 2

        def is_contiguous(self):
            return True

    from types import SimpleNamespace
    out = SimpleNamespace(rows=64, cols=256)
    with pytest.raises(ValueError, match="64 x 256"):
        Q.qlora_quantize(FakeW(), out=out)
