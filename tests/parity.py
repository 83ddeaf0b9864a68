"""Shared helpers of the GPU parity tests: tolerance checks and oracle views."""

import numpy as np
import torch

# Tolerance for bf16 outputs of the forward and backward pass, as the
# acceptance bar states it: relative Frobenius error and max abs/(1+|ref|).
FRO_TOL = 2e-2
MAX_TOL = 1e-2


def f64(t):
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().numpy().astype(np.float64)
    return np.asarray(t, dtype=np.float64)


def assert_close(gpu, ref, name, fro_tol=FRO_TOL, max_tol=MAX_TOL):
    gpu, ref = f64(gpu), f64(ref)
    assert gpu.shape == ref.shape, (name, gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{name}: non-finite values"
    denom = max(np.linalg.norm(ref), 1e-30)
    fro = np.linalg.norm(gpu - ref) / denom
    mx = float(np.max(np.abs(gpu - ref) / (1.0 + np.abs(ref)))) if ref.size else 0.0
    assert fro <= fro_tol and mx <= max_tol, \
        f"{name}: rel Frobenius {fro:.3e} (tol {fro_tol}), max abs/(1+|ref|) {mx:.3e} (tol {max_tol})"
    return fro, mx


def assert_close_scaled(gpu, ref, name, fro_tol=FRO_TOL, max_tol=MAX_TOL):
    """The same bar for fp32 outputs whose size is not O(1) (U, dA, dB): the
    elementwise term is max |gpu - ref| / (rms(ref) + |ref|), i.e. the bf16
    criterion measured in the output's own scale."""
    gpu, ref = f64(gpu), f64(ref)
    assert gpu.shape == ref.shape, (name, gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{name}: non-finite values"
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    if rms == 0.0:
        assert np.array_equal(gpu, ref), f"{name}: reference is zero, output is not"
        return 0.0, 0.0
    fro = np.linalg.norm(gpu - ref) / np.linalg.norm(ref)
    mx = float(np.max(np.abs(gpu - ref) / (rms + np.abs(ref))))
    assert fro <= fro_tol and mx <= max_tol, \
        f"{name}: rel Frobenius {fro:.3e} (tol {fro_tol}), max abs/(rms+|ref|) {mx:.3e} (tol {max_tol})"
    return fro, mx


def oracle_quantised(qt_gpu):
    """The arrays of a library QuantizedWeight as numpy, for comparison."""
    return dict(codes=qt_gpu.codes.cpu().numpy(), scale_codes=qt_gpu.scale_codes.cpu().numpy(),
                factors=qt_gpu.factors.cpu().numpy(), mean=qt_gpu.mean.cpu().numpy())
