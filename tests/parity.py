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


def gpu_available():
    return torch.cuda.is_available()
