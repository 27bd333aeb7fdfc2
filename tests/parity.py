"""Shared helpers for GPU-vs-oracle parity tests.

Tolerances: max-abs |gpu - oracle| <= 2e-2 on O, dQ, dK, dV and <= 1e-3 on
lse, against the fp64 oracle evaluated on the same bf16-rounded inputs.
"""
import numpy as np
import torch

TOL = {"o": 2e-2, "lse": 1e-3, "dq": 2e-2, "dk": 2e-2, "dv": 2e-2}


def np64(t):
    return t.detach().to("cpu", torch.float64).numpy() if torch.is_tensor(t) else np.asarray(t, np.float64)


def max_abs(a, b):
    a, b = np64(a), np64(b)
    assert a.shape == b.shape, (a.shape, b.shape)
    if a.size == 0:
        return 0.0
    assert np.isfinite(a).all(), "non-finite values in GPU output"
    return float(np.abs(a - b).max())


def assert_close(name, gpu, ref, tol=None, ctx=""):
    tol = TOL[name] if tol is None else tol
    err = max_abs(gpu, ref)
    assert err <= tol, f"{name}: max|gpu-oracle| = {err:.3e} > {tol:.1e} {ctx}"
    return err


def assert_close_scaled(name, gpu, ref, tol=None, ctx=""):
    """Max-abs error bounded by tol * max(1, max|ref|).  Used where the
    gradients are not unit-scale (a larger softmax scale, logits in the
    hundreds): bf16 operand rounding is relative (2^-9), so the error of an
    entry grows with the magnitude of the result."""
    tol = TOL[name] if tol is None else tol
    mag = max(1.0, float(np.abs(np64(ref)).max()))
    err = max_abs(gpu, ref)
    assert err <= tol * mag, (f"{name}: max|gpu-oracle| = {err:.3e} > {tol:.1e} * "
                              f"max(1, max|ref| = {mag:.3e}) {ctx}")
    return err


def gpu_available():
    return torch.cuda.is_available()
