"""FP8 (E4M3) forward parity on the GPU: fa_fwd_fp8 through the C ABI against
the fp64 oracle evaluated on the dequantised inputs (e4m3 value x descale).

Tolerance.  S = Q K^T is exact up to fp32 accumulation, so lse keeps the
1e-3 bound.  O carries the E4M3 rounding of P.  With O normalised by the sum
of the rounded p, the error of O_ic is, to first order,
sum_j d_j (v_jc - O_ic), where d_j is the rounding error of the normalised
probability pi_j.  The kernel's p are relative to a running maximum at or
below the row maximum, so their sum is >= 1 and a normalised probability
pi_j >= 2^-6 is an E4M3 normal: |d_j| <= 2^-4 pi_j (half-spacing of a 3-bit
mantissa).  Below that it may be subnormal or flushed: |d_j| <= min(pi_j,
2^-10).  Errors of distinct keys are independent and bounded, so each entry
is checked against 6 standard deviations of that sum (uniform errors: bound
/ sqrt(3) each) plus the bf16 rounding of the output (2^-8 |O|) and 2e-3 for
fp32 accumulation and the f16 partial sums of the normaliser."""
import math

import numpy as np
import pytest
import torch

import oracle
from tiled_attention_20_b200 import inputs
from tests.parity import np64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
SIGMA_E = 2.0 ** -4 / math.sqrt(3.0)


def _fa():
    import tiled_attention_20_b200.fa as fa
    return fa


def _deq(x8, f):
    return x8.to(torch.float64) * f.to(torch.float64)[:, :, None, None]


def _run(B, H, N, causal, seed=0, dist="normal", scale=None):
    fa = _fa()
    q8, k8, v8, fq, fk, fv = inputs.fp8_qkv(B, H, N, 128, seed=seed, dist=dist)
    o, lse = fa.fwd_fp8(q8.to(DEV), k8.to(DEV), v8.to(DEV), fq.to(DEV), fk.to(DEV), fv.to(DEV),
                        scale=scale, causal=causal)
    fa.check_device_errors()
    return _deq(q8, fq), _deq(k8, fk), _deq(v8, fv), o, lse


def _check_head(q, k, v, o, lse, causal, scale, ctx):
    """Full check of one head ([N, d] fp64 inputs, GPU o [N, d], lse [N])."""
    N, d = q.shape
    scale = 1 / math.sqrt(d) if scale is None else scale
    P = oracle.probs(q, k, scale, causal)
    O = P @ v
    o_ref, lse_ref = oracle.fwd(q[None, None], k[None, None], v[None, None], scale, causal)
    np.testing.assert_allclose(O, o_ref[0, 0], rtol=0, atol=1e-10)
    og, lg = np64(o), np64(lse)
    assert np.isfinite(og).all() and np.isfinite(lg).all(), ctx
    lerr = float(np.abs(lg - lse_ref[0, 0]).max())
    assert lerr <= 1e-3, f"lse err {lerr:.2e} {ctx}"
    sd = np.where(P >= 2.0 ** -6, SIGMA_E * P, np.minimum(P, 2.0 ** -10) / math.sqrt(3.0))
    S2 = sd * sd
    var = S2 @ (v * v) - 2 * O * (S2 @ v) + O * O * S2.sum(axis=1, keepdims=True)
    bound = 6 * np.sqrt(np.maximum(var, 0)) + 2.0 ** -8 * np.abs(O) + 2e-3
    err = np.abs(og - O)
    worst = float((err / bound).max())
    assert worst <= 1.0, f"O error exceeds the rounding-model bound by {worst:.2f}x {ctx}"
    return float(err.max()), float(np.sqrt((err ** 2).mean())), worst


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 100, 128, 129, 256, 300, 777, 1024])
def test_fp8_lengths(N, causal):
    q, k, v, o, lse = _run(1, 2, N, causal, seed=N)
    for h in range(2):
        _check_head(q[0, h].numpy(), k[0, h].numpy(), v[0, h].numpy(), o[0, h].cpu(),
                    lse[0, h].cpu(), causal, None, f"N={N} h={h} causal={causal}")


@pytest.mark.parametrize("scale", [0.0, 0.02, 0.3])
def test_fp8_scales(scale):
    q, k, v, o, lse = _run(1, 1, 512, True, seed=3, scale=scale)
    _check_head(q[0, 0].numpy(), k[0, 0].numpy(), v[0, 0].numpy(), o[0, 0].cpu(),
                lse[0, 0].cpu(), True, scale, f"scale={scale}")


def test_fp8_long_context_distribution():
    """Large logits (sigma 3, 1% of rows x8): peaked rows, where P holds a few
    large entries and many tiny ones (E4M3 subnormals)."""
    q, k, v, o, lse = _run(1, 2, 2048, True, seed=1, dist="long_context")
    for h in range(2):
        _check_head(q[0, h].numpy(), k[0, h].numpy(), v[0, h].numpy(), o[0, h].cpu(),
                    lse[0, h].cpu(), True, None, f"long-context h={h}")


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_benchmark_shape_sampled(causal):
    """B=2, H=32, N=4096 (the benchmark workload's shape) in the launch
    configuration the bench times; the oracle checks three heads in full."""
    q, k, v, o, lse = _run(2, 32, 4096, causal, seed=0)
    for b, h in ((0, 0), (1, 17), (1, 31)):
        _check_head(q[b, h].numpy(), k[b, h].numpy(), v[b, h].numpy(), o[b, h].cpu(),
                    lse[b, h].cpu(), causal, None, f"b={b} h={h} causal={causal}")
