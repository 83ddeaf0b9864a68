"""Python binding of libqlora.so (argument marshalling only).

Every function named ``qlora_*`` here calls the C entry point of the same
name in ``include/qlora.h``; tensors are torch tensors (device memory and the
current CUDA stream come from torch), and every step of the computation runs
in the library's CUDA kernels.  A missing library raises immediately: there
is no other implementation to fall back to.
"""

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlora.so")

QLORA_OK = 0
QLORA_ERR_NULL = 1
QLORA_ERR_ALIGN = 2
QLORA_ERR_SHAPE = 3
QLORA_ERR_UNSUPPORTED = 4
QLORA_ERR_NONFINITE = 5
QLORA_ERR_DEVICE_TIMEOUT = 6
QLORA_ERR_CUDA = 7
QLORA_ERR_WORKSPACE = 8

QLORA_F32 = 0
QLORA_BF16 = 1
QLORA_TABLE_NF4 = 0
QLORA_TABLE_UNIFORM = 1

QLORA_KERNEL_QUANTIZE = 0
QLORA_KERNEL_FUSED_FWD = 1
QLORA_KERNEL_FUSED_DGRAD = 2
QLORA_KERNEL_LORA_GEMM = 3
QLORA_KERNEL_MERGE = 4
QLORA_KERNEL_KINDS = 5

_DTYPE = {torch.float32: QLORA_F32, torch.bfloat16: QLORA_BF16}


class qlora_nf4(ctypes.Structure):
    _fields_ = [
        ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
        ("blocksize", ctypes.c_int32), ("dq_blocksize", ctypes.c_int32),
        ("table", ctypes.c_int32), ("reserved", ctypes.c_int32),
        ("codes", ctypes.c_void_p), ("scale_codes", ctypes.c_void_p),
        ("factors", ctypes.c_void_p), ("mean", ctypes.c_void_p),
    ]


class qlora_adapter_opts(ctypes.Structure):
    _fields_ = [
        ("n_adapters", ctypes.c_int32), ("reserved", ctypes.c_int32),
        ("adapter", ctypes.c_void_p), ("dropout_p", ctypes.c_float),
        ("reserved2", ctypes.c_int32), ("keep_mask", ctypes.c_void_p), ("x_drop", ctypes.c_void_p),
    ]


class QloraError(RuntimeError):
    def __init__(self, status, where):
        self.status = int(status)
        super().__init__(f"{where}: {qlora_status_string(status)} (status {status})")


_lib = None


def lib():
    """Load libqlora.so once; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m bit_nf4_quantized_17_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        i32, i64, sz, vp, f32 = (ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t,
                                 ctypes.c_void_p, ctypes.c_float)
        psz = ctypes.POINTER(ctypes.c_size_t)
        pq = ctypes.POINTER(qlora_nf4)
        po = ctypes.POINTER(qlora_adapter_opts)
        sig = {
            "qlora_status_string": (ctypes.c_char_p, [ctypes.c_int]),
            "qlora_levels": (ctypes.c_int, [i32, ctypes.POINTER(ctypes.c_float)]),
            "qlora_nf4_sizes": (ctypes.c_int, [i64, i64, i32, i32, psz, psz, psz, psz, psz]),
            "qlora_quantize": (ctypes.c_int, [vp, i32, pq, vp, sz, vp]),
            "qlora_dequantize": (ctypes.c_int, [pq, vp, i32, vp]),
            "qlora_linear_workspace": (ctypes.c_int, [i64, i64, i64, i32, psz, psz]),
            "qlora_linear_fwd": (ctypes.c_int, [pq, vp, vp, i32, f32, vp, i64, vp, vp, vp, sz, vp]),
            "qlora_linear_bwd": (ctypes.c_int, [pq, vp, vp, i32, f32, vp, vp, vp, i64, vp, vp, vp,
                                                i32, vp, sz, vp]),
            "qlora_linear_fwd_multi": (ctypes.c_int, [pq, vp, vp, i32, i32, f32, vp, vp, i64, vp,
                                                      vp, vp, sz, vp]),
            "qlora_linear_bwd_multi": (ctypes.c_int, [pq, vp, vp, i32, i32, f32, vp, vp, vp, vp,
                                                      i64, vp, vp, vp, i32, vp, sz, vp]),
            "qlora_linear_fwd_ex": (ctypes.c_int, [pq, vp, vp, i32, f32, po, vp, i64, vp, vp, vp,
                                                   sz, vp]),
            "qlora_linear_bwd_ex": (ctypes.c_int, [pq, vp, vp, i32, f32, po, vp, vp, vp, i64, vp,
                                                   vp, vp, i32, vp, sz, vp]),
            "qlora_check": (ctypes.c_int, [vp, vp]),
            "qlora_selftest_timeout": (ctypes.c_int, [i64, vp, vp]),
            "qlora_merge": (ctypes.c_int, [pq, vp, vp, i32, f32, vp, vp]),
            "qlora_merge_dense": (ctypes.c_int, [vp, i64, i64, vp, vp, i32, f32, vp, vp]),
            "qlora_paged_alloc": (ctypes.c_int, [ctypes.c_size_t, ctypes.POINTER(ctypes.c_void_p)]),
            "qlora_paged_prefetch": (ctypes.c_int, [vp, ctypes.c_size_t, i32, vp]),
            "qlora_paged_free": (ctypes.c_int, [vp]),
            "qlora_adamw": (ctypes.c_int, [vp, vp, vp, vp, vp, i64, i32, f32, f32, f32, f32, f32,
                                           f32, vp]),
            "qlora_launch_count": (ctypes.c_uint64, []),
            "qlora_timing_begin": (ctypes.c_int, [ctypes.c_uint32, i32]),
            "qlora_timing_end": (ctypes.c_int, [ctypes.POINTER(ctypes.c_float),
                                                ctypes.POINTER(ctypes.c_int32)]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ok(status, where):
    if status != QLORA_OK:
        raise QloraError(status, where)


def qlora_status_string(status):
    return lib().qlora_status_string(int(status)).decode()


def qlora_levels(table=QLORA_TABLE_NF4):
    out = (ctypes.c_float * 16)()
    _ok(lib().qlora_levels(table, out), "qlora_levels")
    return list(out)


def qlora_nf4_sizes(rows, cols, blocksize=64, dq_blocksize=256):
    vals = [ctypes.c_size_t() for _ in range(5)]
    _ok(lib().qlora_nf4_sizes(rows, cols, blocksize, dq_blocksize,
                              *[ctypes.byref(v) for v in vals]), "qlora_nf4_sizes")
    keys = ("codes", "scale_codes", "factors", "mean", "workspace")
    return {k: v.value for k, v in zip(keys, vals)}


def qlora_linear_workspace(M, N, K, r):
    f, b = ctypes.c_size_t(), ctypes.c_size_t()
    _ok(lib().qlora_linear_workspace(M, N, K, r, ctypes.byref(f), ctypes.byref(b)),
        "qlora_linear_workspace")
    return f.value, b.value


def _check_linear(q, M, rt, **tensors):
    """The library sees only pointers: check each tensor's shape, dtype, device and
    layout here, so that a mismatch raises instead of reading or writing past a buffer.
    Names: A, B, X, Y, U, dY, dX, dA, dB, adapter, keep_mask, x_drop (None = absent)."""
    K, N = q.cols, q.rows
    spec = {
        "A": ((rt, K), torch.bfloat16), "B": ((N, rt), torch.bfloat16),
        "X": ((M, K), torch.bfloat16), "Y": ((M, N), torch.bfloat16),
        "U": ((M, rt), torch.float32), "dY": ((M, N), torch.bfloat16),
        "dX": ((M, K), torch.bfloat16), "dA": ((rt, K), torch.float32),
        "dB": ((N, rt), torch.float32), "adapter": ((M,), torch.int32),
        "keep_mask": ((M, K // 8), torch.uint8), "x_drop": ((M, K), torch.bfloat16),
    }
    for name, t in tensors.items():
        if t is None:
            continue
        shape, dtype = spec[name]
        if tuple(t.shape) != shape or t.dtype != dtype or not t.is_contiguous() or not t.is_cuda:
            raise ValueError(f"{name}: expected a contiguous CUDA {dtype} tensor of shape "
                             f"{shape}, got {t.dtype} {tuple(t.shape)} on {t.device}"
                             f"{'' if t.is_contiguous() else ', not contiguous'}")


def _workspace(nbytes, device):
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


@dataclass
class QuantizedWeight:
    """Caller-owned device arrays of one quantised weight (see qlora_nf4)."""
    rows: int
    cols: int
    blocksize: int
    dq_blocksize: int
    table: int
    codes: torch.Tensor
    scale_codes: torch.Tensor
    factors: torch.Tensor
    mean: torch.Tensor

    @classmethod
    def empty(cls, rows, cols, blocksize=64, dq_blocksize=256, table=QLORA_TABLE_NF4,
              device="cuda"):
        sz = qlora_nf4_sizes(rows, cols, blocksize, dq_blocksize)
        return cls(rows, cols, blocksize, dq_blocksize, table,
                   torch.empty(sz["codes"], dtype=torch.uint8, device=device),
                   torch.empty(max(sz["scale_codes"], 1), dtype=torch.int8, device=device),
                   torch.empty(sz["factors"] // 4, dtype=torch.float32, device=device),
                   torch.empty(max(sz["mean"] // 4, 1), dtype=torch.float32, device=device))

    @property
    def struct(self):
        return qlora_nf4(self.rows, self.cols, self.blocksize, self.dq_blocksize, self.table, 0,
                         self.codes.data_ptr(), self.scale_codes.data_ptr(),
                         self.factors.data_ptr(), self.mean.data_ptr())

    @property
    def nbytes(self):
        sz = qlora_nf4_sizes(self.rows, self.cols, self.blocksize, self.dq_blocksize)
        return sz["codes"] + sz["scale_codes"] + sz["factors"] + sz["mean"]


def qlora_quantize(W, blocksize=64, dq_blocksize=256, table=QLORA_TABLE_NF4, out=None,
                   workspace=None, stream=None, check=True):
    """Quantise a 2-D fp32/bf16 CUDA tensor; returns a QuantizedWeight."""
    assert W.is_cuda and W.dim() == 2 and W.is_contiguous() and W.dtype in _DTYPE
    rows, cols = W.shape
    q = out or QuantizedWeight.empty(rows, cols, blocksize, dq_blocksize, table, W.device)
    if (q.rows, q.cols) != (rows, cols):
        raise ValueError(f"out holds a {q.rows} x {q.cols} weight, W is {rows} x {cols}")
    if workspace is None:
        workspace = _workspace(qlora_nf4_sizes(rows, cols, blocksize, dq_blocksize)["workspace"],
                               W.device)
    st = q.struct
    _ok(lib().qlora_quantize(_ptr(W), _DTYPE[W.dtype], ctypes.byref(st), _ptr(workspace),
                             workspace.numel(), _stream(stream)), "qlora_quantize")
    if check:
        qlora_check(workspace, stream)
    return q


def qlora_dequantize(q, dtype=torch.float32, out=None, stream=None):
    out = out if out is not None else torch.empty((q.rows, q.cols), dtype=dtype,
                                                  device=q.codes.device)
    if tuple(out.shape) != (q.rows, q.cols) or out.dtype not in _DTYPE or not out.is_contiguous():
        raise ValueError(f"out: expected a contiguous fp32 or bf16 tensor of shape "
                         f"{(q.rows, q.cols)}")
    st = q.struct
    _ok(lib().qlora_dequantize(ctypes.byref(st), _ptr(out), _DTYPE[out.dtype], _stream(stream)),
        "qlora_dequantize")
    return out


def qlora_linear_fwd(q, A, B, alpha, X, Y=None, U_save=None, workspace=None, stream=None,
                     check=False):
    """Y = X W^T + (alpha/r) (X A^T) B^T.  Returns Y (and fills U_save if given).
    check=True synchronises and raises on a device-side error status."""
    M = X.shape[0]
    r = A.shape[0]
    if Y is None:
        Y = torch.empty((M, q.rows), dtype=torch.bfloat16, device=X.device)
    _check_linear(q, M, r, A=A, B=B, X=X, Y=Y, U=U_save)
    if workspace is None:
        workspace = _workspace(qlora_linear_workspace(M, q.rows, q.cols, r)[0], X.device)
    st = q.struct
    _ok(lib().qlora_linear_fwd(ctypes.byref(st), _ptr(A), _ptr(B), r, float(alpha), _ptr(X), M,
                               _ptr(Y), _ptr(U_save), _ptr(workspace), workspace.numel(),
                               _stream(stream)), "qlora_linear_fwd")
    if check:
        qlora_check(workspace, stream)
    return Y


def qlora_linear_fwd_multi(q, A, B, r, alpha, adapter, X, Y=None, U_save=None, workspace=None,
                           stream=None, check=False):
    """Several rank-r adapters stacked along the rank (A: (n r) x d_in, B:
    d_out x (n r)); token m uses adapter adapter[m] (int32, -1 = none)."""
    M = X.shape[0]
    rt = A.shape[0]
    if rt % r:
        raise ValueError(f"A has {rt} rows: not a stack of rank-{r} adapters")
    n = rt // r
    if Y is None:
        Y = torch.empty((M, q.rows), dtype=torch.bfloat16, device=X.device)
    _check_linear(q, M, rt, A=A, B=B, X=X, Y=Y, U=U_save, adapter=adapter)
    if workspace is None:
        workspace = _workspace(qlora_linear_workspace(M, q.rows, q.cols, rt)[0], X.device)
    st = q.struct
    _ok(lib().qlora_linear_fwd_multi(ctypes.byref(st), _ptr(A), _ptr(B), n, r, float(alpha),
                                     _ptr(adapter), _ptr(X), M, _ptr(Y), _ptr(U_save),
                                     _ptr(workspace), workspace.numel(), _stream(stream)),
        "qlora_linear_fwd_multi")
    if check:
        qlora_check(workspace, stream)
    return Y


def qlora_linear_bwd_multi(q, A, B, r, alpha, adapter, X, U, dY, dX=None, dA=None, dB=None,
                           accumulate=False, want_dx=True, workspace=None, stream=None,
                           check=False):
    """Backward of qlora_linear_fwd_multi; dA and dB in the stacked layouts."""
    M = X.shape[0]
    rt = A.shape[0]
    if rt % r:
        raise ValueError(f"A has {rt} rows: not a stack of rank-{r} adapters")
    n = rt // r
    dev = X.device
    if want_dx and dX is None:
        dX = torch.empty((M, q.cols), dtype=torch.bfloat16, device=dev)
    if dA is None:
        dA = torch.empty((rt, q.cols), dtype=torch.float32, device=dev)
    if dB is None:
        dB = torch.empty((q.rows, rt), dtype=torch.float32, device=dev)
    _check_linear(q, M, rt, A=A, B=B, X=X, U=U, dY=dY, dX=dX if want_dx else None, dA=dA, dB=dB,
                  adapter=adapter)
    if workspace is None:
        workspace = _workspace(qlora_linear_workspace(M, q.rows, q.cols, rt)[1], dev)
    st = q.struct
    _ok(lib().qlora_linear_bwd_multi(ctypes.byref(st), _ptr(A), _ptr(B), n, r, float(alpha),
                                     _ptr(adapter), _ptr(X), _ptr(U), _ptr(dY), M,
                                     _ptr(dX) if want_dx else None, _ptr(dA), _ptr(dB),
                                     1 if accumulate else 0, _ptr(workspace), workspace.numel(),
                                     _stream(stream)), "qlora_linear_bwd_multi")
    if check:
        qlora_check(workspace, stream)
    return dX, dA, dB


def dropout_keep_mask(M, K, p, generator=None, device="cuda"):
    """A keep mask for LoRA dropout, drawn with torch's generator (the random
    draw is an input of the layer): M x K/8 uint8, bit (k % 8) of byte
    [m][k / 8] set = keep X[m][k], each kept with probability 1 - p."""
    keep = torch.rand((M, K // 8, 8), generator=generator, device=device) >= p
    weights = (1 << torch.arange(8, device=device, dtype=torch.int32))
    return (keep.to(torch.int32) * weights).sum(-1).to(torch.uint8).contiguous()


def _opts(r, A, adapter, p, keep_mask, x_drop):
    o = qlora_adapter_opts()
    rt = A.shape[0]
    if rt % r:
        raise ValueError(f"A has {rt} rows: not a stack of rank-{r} adapters")
    o.n_adapters = rt // r
    o.adapter = adapter.data_ptr() if adapter is not None else None
    o.dropout_p = float(p)
    o.keep_mask = keep_mask.data_ptr() if keep_mask is not None else None
    o.x_drop = x_drop.data_ptr() if x_drop is not None else None
    return o


def qlora_linear_fwd_ex(q, A, B, r, alpha, X, adapter=None, p=0.0, keep_mask=None, x_drop=None,
                        Y=None, U_save=None, workspace=None, stream=None, check=False):
    """Forward with optional per-token adapters (A, B stacked along the rank)
    and LoRA dropout (keep_mask from dropout_keep_mask; x_drop receives
    X (.) D and must be passed again to the backward)."""
    M = X.shape[0]
    rt = A.shape[0]
    o = _opts(r, A, adapter, p, keep_mask, x_drop)
    if Y is None:
        Y = torch.empty((M, q.rows), dtype=torch.bfloat16, device=X.device)
    _check_linear(q, M, rt, A=A, B=B, X=X, Y=Y, U=U_save, adapter=adapter, keep_mask=keep_mask,
                  x_drop=x_drop)
    if workspace is None:
        workspace = _workspace(qlora_linear_workspace(M, q.rows, q.cols, rt)[0], X.device)
    st = q.struct
    _ok(lib().qlora_linear_fwd_ex(ctypes.byref(st), _ptr(A), _ptr(B), r, float(alpha),
                                  ctypes.byref(o), _ptr(X), M, _ptr(Y), _ptr(U_save),
                                  _ptr(workspace), workspace.numel(), _stream(stream)),
        "qlora_linear_fwd_ex")
    if check:
        qlora_check(workspace, stream)
    return Y


def qlora_linear_bwd_ex(q, A, B, r, alpha, X, U, dY, adapter=None, p=0.0, keep_mask=None,
                        x_drop=None, dX=None, dA=None, dB=None, accumulate=False, want_dx=True,
                        workspace=None, stream=None, check=False):
    """Backward of qlora_linear_fwd_ex (same adapter ids, mask and x_drop)."""
    M = X.shape[0]
    rt = A.shape[0]
    dev = X.device
    o = _opts(r, A, adapter, p, keep_mask, x_drop)
    if want_dx and dX is None:
        dX = torch.empty((M, q.cols), dtype=torch.bfloat16, device=dev)
    if dA is None:
        dA = torch.empty((rt, q.cols), dtype=torch.float32, device=dev)
    if dB is None:
        dB = torch.empty((q.rows, rt), dtype=torch.float32, device=dev)
    _check_linear(q, M, rt, A=A, B=B, X=X, U=U, dY=dY, dX=dX if want_dx else None, dA=dA, dB=dB,
                  adapter=adapter, keep_mask=keep_mask, x_drop=x_drop)
    if workspace is None:
        workspace = _workspace(qlora_linear_workspace(M, q.rows, q.cols, rt)[1], dev)
    st = q.struct
    _ok(lib().qlora_linear_bwd_ex(ctypes.byref(st), _ptr(A), _ptr(B), r, float(alpha),
                                  ctypes.byref(o), _ptr(X), _ptr(U), _ptr(dY), M,
                                  _ptr(dX) if want_dx else None, _ptr(dA), _ptr(dB),
                                  1 if accumulate else 0, _ptr(workspace), workspace.numel(),
                                  _stream(stream)), "qlora_linear_bwd_ex")
    if check:
        qlora_check(workspace, stream)
    return dX, dA, dB


def qlora_linear_bwd(q, A, B, alpha, X, U, dY, dX=None, dA=None, dB=None, accumulate=False,
                     want_dx=True, workspace=None, stream=None, check=False):
    """Returns (dX, dA, dB); W gets no gradient.
    check=True synchronises and raises on a device-side error status."""
    M = X.shape[0]
    r = A.shape[0]
    dev = X.device
    if want_dx and dX is None:
        dX = torch.empty((M, q.cols), dtype=torch.bfloat16, device=dev)
    if dA is None:
        dA = torch.empty((r, q.cols), dtype=torch.float32, device=dev)
    if dB is None:
        dB = torch.empty((q.rows, r), dtype=torch.float32, device=dev)
    _check_linear(q, M, r, A=A, B=B, X=X, U=U, dY=dY, dX=dX if want_dx else None, dA=dA, dB=dB)
    if workspace is None:
        workspace = _workspace(qlora_linear_workspace(M, q.rows, q.cols, r)[1], dev)
    st = q.struct
    _ok(lib().qlora_linear_bwd(ctypes.byref(st), _ptr(A), _ptr(B), r, float(alpha), _ptr(X),
                               _ptr(U), _ptr(dY), M, _ptr(dX) if want_dx else None, _ptr(dA),
                               _ptr(dB), 1 if accumulate else 0, _ptr(workspace),
                               workspace.numel(), _stream(stream)), "qlora_linear_bwd")
    if check:
        qlora_check(workspace, stream)
    return dX, dA, dB


def qlora_launch_count():
    return int(lib().qlora_launch_count())


def qlora_merge(q, A, B, alpha, out=None, stream=None):
    """W_merged = bf16(dequant(W) + (alpha / r) B A) as a new (or given) bf16 tensor."""
    r = A.shape[0]
    out = out if out is not None else torch.empty((q.rows, q.cols), dtype=torch.bfloat16,
                                                  device=A.device)
    _check_linear(q, 0, r, A=A, B=B)
    if (tuple(out.shape) != (q.rows, q.cols) or out.dtype != torch.bfloat16
            or not out.is_contiguous()):
        raise ValueError(f"out: expected a contiguous bf16 tensor of shape {(q.rows, q.cols)}")
    st = q.struct
    _ok(lib().qlora_merge(ctypes.byref(st), _ptr(A), _ptr(B), r, float(alpha), _ptr(out),
                          _stream(stream)), "qlora_merge")
    return out


def qlora_merge_dense(W, A, B, alpha, out=None, stream=None):
    """bf16(W + (alpha / r) B A) for a dense bf16 W; out=W works in place, and
    -alpha takes a merged adapter out again."""
    r = A.shape[0]
    rows, cols = W.shape
    out = out if out is not None else torch.empty_like(W)
    for name, t, shape in (("W", W, (rows, cols)), ("A", A, (r, cols)), ("B", B, (rows, r)),
                           ("out", out, (rows, cols))):
        if tuple(t.shape) != shape or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError(f"{name}: expected a contiguous bf16 tensor of shape {shape}")
    _ok(lib().qlora_merge_dense(_ptr(W), rows, cols, _ptr(A), _ptr(B), r, float(alpha), _ptr(out),
                                _stream(stream)), "qlora_merge_dense")
    return out


def qlora_adamw(param, grad, m, v, step, lr, beta1=0.9, beta2=0.999, eps=1e-8,
                weight_decay=0.0, grad_scale=1.0, param_bf16=None, stream=None):
    """One AdamW step in place over flat fp32 tensors (param, m, v updated);
    param_bf16, if given, receives bf16(param)."""
    n = param.numel()
    for t in (param, grad, m, v):
        assert t.dtype == torch.float32 and t.is_contiguous() and t.numel() == n
    _ok(lib().qlora_adamw(_ptr(param), _ptr(param_bf16), _ptr(grad), _ptr(m), _ptr(v), n,
                          int(step), float(lr), float(beta1), float(beta2), float(eps),
                          float(weight_decay), float(grad_scale), _stream(stream)), "qlora_adamw")


class _PagedBlock:
    """Owner of one qlora_paged_alloc block, exposed to torch through the CUDA
    array interface; the block is freed when the last tensor on it goes."""

    def __init__(self, numel, dtype):
        self.nbytes = int(numel) * torch.empty((), dtype=dtype).element_size()
        ptr = ctypes.c_void_p()
        _ok(lib().qlora_paged_alloc(self.nbytes, ctypes.byref(ptr)), "qlora_paged_alloc")
        self.ptr = ptr.value
        typestr = {torch.float32: "<f4", torch.uint8: "|u1"}[dtype]
        self.__cuda_array_interface__ = {
            "shape": (int(numel),), "typestr": typestr, "data": (self.ptr, False),
            "version": 3, "strides": None, "stream": None}

    def __del__(self):
        if getattr(self, "ptr", None) and _lib is not None:
            _lib.qlora_paged_free(ctypes.c_void_p(self.ptr))
            self.ptr = None


def qlora_paged_empty(numel, dtype=torch.float32):
    """A zero-filled 1-D tensor of `numel` elements in managed (paged) memory
    from qlora_paged_alloc; it keeps its block alive."""
    if dtype not in (torch.float32, torch.uint8):
        raise ValueError("paged tensors are fp32 or uint8")
    return torch.as_tensor(_PagedBlock(numel, dtype), device="cuda")


def qlora_paged_prefetch(t, to_device=True, stream=None):
    """Enqueue a migration of tensor `t`'s pages to the current GPU or to host memory."""
    _ok(lib().qlora_paged_prefetch(_ptr(t), t.numel() * t.element_size(), 1 if to_device else 0,
                                   _stream(stream)), "qlora_paged_prefetch")


def qlora_timing_begin(kinds, max_launches=4096):
    """Start timing every launch of the given kernel kinds (QLORA_KERNEL_*)."""
    mask = 0
    for k in kinds:
        mask |= 1 << int(k)
    _ok(lib().qlora_timing_begin(mask, int(max_launches)), "qlora_timing_begin")


def qlora_timing_end():
    """Stop timing; {kind: (total ms, launches)} for every kind."""
    ms = (ctypes.c_float * QLORA_KERNEL_KINDS)()
    n = (ctypes.c_int32 * QLORA_KERNEL_KINDS)()
    _ok(lib().qlora_timing_end(ms, n), "qlora_timing_end")
    return {k: (float(ms[k]), int(n[k])) for k in range(QLORA_KERNEL_KINDS)}


def qlora_selftest_timeout(limit_cycles, workspace, stream=None):
    """Enqueue the library's bounded-wait failure path on purpose (see the header)."""
    _ok(lib().qlora_selftest_timeout(int(limit_cycles), _ptr(workspace), _stream(stream)),
        "qlora_selftest_timeout")


def qlora_check(workspace, stream=None):
    _ok(lib().qlora_check(_ptr(workspace), _stream(stream)), "qlora_check")
