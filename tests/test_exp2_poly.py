"""The kernel's polynomial 2^x (used for part of the softmax exponentials on
the FMA pipe) against exact 2^x: its coefficients are read from the CUDA
header and evaluated exactly as the kernel does, in fp32 with the same
rounding steps, then compared in fp64."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "tiled_attention_20_b200", "csrc", "sm100.cuh")


def _coeffs():
    text = open(HDR).read()
    vals = {}
    for k in range(4):
        m = re.search(rf"kExp2C{k}\s*=\s*([0-9.eE+-]+)f", text)
        assert m, f"kExp2C{k} not found"
        vals[k] = np.float32(float(m.group(1)))
    return [vals[k] for k in range(4)]


def _poly_exp2_f32(x):
    """fp32 emulation of exp2_poly2: clamp, 1.5*2^23 shifter rounding,
    Horner, integer add of round(x) into the exponent field."""
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    sh = np.float32(12582912.0)
    t = (x + sh).astype(np.float32)
    n = (t - sh).astype(np.float32)
    f = (x - n).astype(np.float32)
    q = (c3 * f + c2).astype(np.float32)   # separate rounding per step is at
    q = (q * f + c1).astype(np.float32)    # least as bad as a fused fma, so the
    q = (q * f + c0).astype(np.float32)    # bound below also covers the kernel
    bits = q.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    x = np.linspace(-125.0, 8.0, 2_000_003, dtype=np.float64).astype(np.float32)
    got = _poly_exp2_f32(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 8e-5, rel.max()      # below 2^-13.6; bf16 keeps 2^-9


def test_integer_and_half_points():
    x = np.arange(-124, 9, dtype=np.float32)
    got = _poly_exp2_f32(x).astype(np.float64)
    np.testing.assert_allclose(got, np.exp2(x.astype(np.float64)), rtol=8e-5)
    got = _poly_exp2_f32(x + np.float32(0.5)).astype(np.float64)
    np.testing.assert_allclose(got, np.exp2(x.astype(np.float64) + 0.5), rtol=8e-5)


def test_clamp_keeps_results_normal():
    x = np.array([-np.inf, -1e30, -200.0, -125.0, -124.6], dtype=np.float32)
    got = _poly_exp2_f32(x)
    assert np.all(np.isfinite(got)) and np.all(got > 0)
    assert np.all(got <= np.float32(2.0 ** -124))
    assert np.all(got >= np.float32(2.0 ** -126))  # a normal fp32, never a wrapped exponent
