"""Shared helpers for GPU-vs-oracle parity tests.

Tolerances: max-abs |gpu - oracle| <= 2e-2 on O, dQ, dK, dV and <= 1e-3 on
lse, against the fp64 oracle evaluated on the same bf16-rounded inputs.
"""
import json
import os

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


def assert_close_bf16_out(name, gpu, ref, tol=None, ctx=""):
    """For results stored in bf16: |gpu - oracle| <= tol + 2^-8 |oracle| per
    element.  Rounding a value x to bf16 (8 significant bits, round to
    nearest even) moves it by at most half a unit in the last place, which is
    at most 2^-8 |x|; a gradient of magnitude 8 or more can therefore not be
    stored within an absolute 2e-2 at all.  Returns the largest excess of
    |gpu - oracle| over 2^-8 |oracle| (<= tol)."""
    tol = TOL[name] if tol is None else tol
    a, r = np64(gpu), np64(ref)
    assert a.shape == r.shape, (a.shape, r.shape)
    assert np.isfinite(a).all(), "non-finite values in GPU output"
    excess = float((np.abs(a - r) - 2.0 ** -8 * np.abs(r)).max()) if a.size else 0.0
    assert excess <= tol, (f"{name}: max(|gpu-oracle| - 2^-8|oracle|) = {excess:.3e} > "
                           f"{tol:.1e} {ctx}")
    return excess


def gpu_available():
    return torch.cuda.is_available()


def record(**fields):
    """Appends one JSON line of measured errors to the file named by the
    FA_PARITY_RECORD environment variable (no-op when it is unset), so a GPU
    run can keep the numbers a tolerance decision rests on."""
    path = os.environ.get("FA_PARITY_RECORD")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(fields) + "\n")
