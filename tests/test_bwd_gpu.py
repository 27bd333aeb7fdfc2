"""Backward parity on the GPU: fa_bwd through the C ABI (on the forward's own
O and lse) against the fp64 oracle's exact gradient."""
import numpy as np
import pytest
import torch

import oracle
from tiled_attention_20_b200 import inputs
from tests.parity import assert_close, assert_close_scaled, np64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _fa():
    import tiled_attention_20_b200.fa as fa
    return fa


def _run(B, H, N, d, causal, seed=0, dist="normal", grad_dtype=torch.bfloat16, scale=None):
    fa = _fa()
    q, k, v, dO = inputs.qkv_do(B, H, N, d, seed=seed, dist=dist)
    qd, kd, vd, dOd = (t.to(DEV) for t in (q, k, v, dO))
    o, lse = fa.fwd(qd, kd, vd, scale=scale, causal=causal)
    dq, dk, dv = fa.bwd(qd, kd, vd, o, dOd, lse, scale=scale, causal=causal, grad_dtype=grad_dtype)
    fa.check_device_errors()
    return (q, k, v, dO), (o, lse), (dq, dk, dv)


def _check(B, H, N, d, causal, seed=0, dist="normal", grad_dtype=torch.bfloat16, scale=None,
           scaled_tol=False):
    (q, k, v, dO), (o, lse), (dq, dk, dv) = _run(B, H, N, d, causal, seed, dist, grad_dtype, scale)
    dq_r, dk_r, dv_r, _, _ = oracle.bwd(q, k, v, dO, scale=scale, causal=causal)
    ctx = f"B={B} H={H} N={N} d={d} causal={causal}"
    cmp = assert_close_scaled if scaled_tol else assert_close
    e = {"dq": cmp("dq", dq, dq_r, ctx=ctx),
         "dk": cmp("dk", dk, dk_r, ctx=ctx),
         "dv": cmp("dv", dv, dv_r, ctx=ctx)}
    return e


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 2, 63, 64, 65, 127, 128, 129, 200, 255, 256, 300, 513])
def test_ragged_lengths(N, d, causal):
    _check(1, 2, N, d, causal, seed=N + d)


@pytest.mark.parametrize("causal", [False, True])
def test_mid_config(causal):
    """B=4, H=16, N=1024, d=64 forward and backward, full oracle."""
    (q, k, v, dO), (o, lse), (dq, dk, dv) = _run(4, 16, 1024, 64, causal)
    o_r, lse_r = oracle.fwd(q, k, v, causal=causal)
    assert_close("o", o, o_r)
    assert_close("lse", lse, lse_r)
    dq_r, dk_r, dv_r, _, _ = oracle.bwd(q, k, v, dO, causal=causal)
    assert_close("dq", dq, dq_r)
    assert_close("dk", dk, dk_r)
    assert_close("dv", dv, dv_r)


@pytest.mark.parametrize("d", [64, 128])
def test_fp32_gradients(d):
    _check(2, 2, 333, d, True, seed=7, grad_dtype=torch.float32)
    _check(1, 3, 190, d, False, seed=8, grad_dtype=torch.float32)


def test_scale_argument():
    """Non-default scales.  A larger scale sharpens the softmax and grows the
    gradients (max|dQ| about 5.7 here), and bf16 operand rounding is relative,
    so the bound is scaled by the magnitude of the result."""
    _check(1, 2, 257, 64, True, seed=11, scale=0.3, scaled_tol=True)
    _check(1, 2, 257, 64, True, seed=11, scale=0.3, grad_dtype=torch.float32, scaled_tol=True)
    _check(1, 2, 257, 128, False, seed=12, scale=0.05)


def test_long_context_distribution_small():
    """Q, K ~ N(0, 3) with 1% of rows x8: logits in the hundreds and gradients
    far from unit scale, so the bound is scaled by the result's magnitude."""
    for d in (64, 128):
        _check(1, 2, 1100, d, True, seed=5, dist="long_context", scaled_tol=True)


@pytest.mark.parametrize("causal", [False, True])
def test_gradient_sum_rules_on_gpu(causal):
    """Key-shift invariance gives sum_j dK_j = 0; rows of P summing to one give
    sum_j dV_j = sum_i dO_i.  Checked per head and column on fp32 gradient
    outputs, with bounds from the rounding model of the kernel: the bf16
    operands P and dS carry a relative error of at most 2^-9 each, and D is
    formed from the bf16 output O, so sum_j dS_ij is off by at most
    2^-9 sum_c |dO_ic O_ic|.  The bounds below are those, doubled."""
    (q, k, v, dO), (o, _), (dq, dk, dv) = _run(2, 4, 700, 128, causal, seed=3,
                                               grad_dtype=torch.float32)
    scale = 1 / np.sqrt(128)
    dk64, dv64, dO64, q64, o64 = np64(dk), np64(dv), np64(dO), np64(q), np64(o)
    u = 2.0 ** -9
    dd = np.abs(dO64 * o64).sum(axis=3, keepdims=True)          # [B,H,N,1]
    bound_k = 2 * (u * np.abs(dk64).sum(axis=2) + scale * u * (dd * np.abs(q64)).sum(axis=2))
    assert (np.abs(dk64.sum(axis=2)) <= bound_k).all(), np.abs(dk64.sum(axis=2)).max()
    bound_v = 2 * u * np.abs(dO64).sum(axis=2) + 1e-6
    assert (np.abs(dv64.sum(axis=2) - dO64.sum(axis=2)) <= bound_v).all()


def test_workspace_contents_do_not_matter():
    fa = _fa()
    q, k, v, dO = (t.to(DEV) for t in inputs.qkv_do(1, 2, 300, 128, seed=2))
    o, lse = fa.fwd(q, k, v, causal=True)
    ws = torch.full((fa.workspace_size(1, 2, 300, 128),), 0x7F, dtype=torch.uint8, device=DEV)
    a = fa.bwd(q, k, v, o, dO, lse, causal=True, workspace=ws, grad_dtype=torch.float32)
    ws.fill_(0xFF)
    b = fa.bwd(q, k, v, o, dO, lse, causal=True, workspace=ws, grad_dtype=torch.float32)
    fa.check_device_errors()
    for x, y in zip(a, b):
        assert torch.allclose(x, y, atol=1e-5, rtol=0)
