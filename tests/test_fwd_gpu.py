"""Forward parity on the GPU: fa_fwd through the C ABI against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
from tiled_attention_20_b200 import inputs
from tests.parity import assert_close, np64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _fa():
    import tiled_attention_20_b200.fa as fa
    return fa


def _run(B, H, N, d, causal, seed=0, dist="normal", scale=None):
    fa = _fa()
    q, k, v, _ = inputs.qkv_do(B, H, N, d, seed=seed, dist=dist)
    o, lse = fa.fwd(q.to(DEV), k.to(DEV), v.to(DEV), scale=scale, causal=causal)
    fa.check_device_errors()
    return q, k, v, o, lse


@pytest.mark.parametrize("causal", [False, True])
def test_small_forward_config(causal):
    """B=1, H=2, N=256, d=64 (the small forward-only workload), full oracle."""
    q, k, v, o, lse = _run(1, 2, 256, 64, causal)
    o_ref, lse_ref = oracle.fwd(q, k, v, causal=causal)
    assert_close("o", o, o_ref)
    assert_close("lse", lse, lse_ref)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 2, 63, 127, 128, 129, 255, 256, 257, 300, 513, 1000])
def test_ragged_lengths(N, d, causal):
    q, k, v, o, lse = _run(1, 3, N, d, causal, seed=N)
    o_ref, lse_ref = oracle.fwd(q, k, v, causal=causal)
    assert_close("o", o, o_ref, ctx=f"N={N} d={d} causal={causal}")
    assert_close("lse", lse, lse_ref, ctx=f"N={N} d={d} causal={causal}")


@pytest.mark.parametrize("causal", [False, True])
def test_mid_config_forward(causal):
    """B=4, H=16, N=1024, d=64, full oracle."""
    q, k, v, o, lse = _run(4, 16, 1024, 64, causal)
    o_ref, lse_ref = oracle.fwd(q, k, v, causal=causal)
    assert_close("o", o, o_ref)
    assert_close("lse", lse, lse_ref)


def test_causal_row0_is_v0_bit_exact():
    """Row 0 of causal attention sees only key 0, so O_0 = bf16(V_0) exactly."""
    for d in (64, 128):
        q, k, v, o, lse = _run(2, 4, 300, d, True, seed=5)
        assert torch.equal(o[:, :, 0].cpu(), v[:, :, 0])
        s00 = (q[:, :, 0].double() * k[:, :, 0].double()).sum(-1) / np.sqrt(d)
        assert np.abs(np64(lse[:, :, 0]) - s00.numpy()).max() < 1e-4


@pytest.mark.parametrize("causal", [False, True])
def test_uniform_scores_mean_of_v(causal):
    fa = _fa()
    B, H, N, d = 1, 2, 333, 128
    _, k, v, _ = inputs.qkv_do(B, H, N, d, seed=9)
    q = torch.zeros_like(k)
    o, lse = fa.fwd(q.to(DEV), k.to(DEV), v.to(DEV), causal=causal)
    fa.check_device_errors()
    vv = np64(v)
    if causal:
        ref = np.cumsum(vv, axis=2) / np.arange(1, N + 1)[None, None, :, None]
        lref = np.log(np.arange(1, N + 1))[None, None, :]
    else:
        ref = np.broadcast_to(vv.mean(axis=2, keepdims=True), vv.shape)
        lref = np.full((B, H, N), np.log(N))
    assert_close("o", o, ref)
    assert_close("lse", lse, np.broadcast_to(lref, (B, H, N)))


def test_scale_argument_and_zero_scale():
    q, k, v, o, lse = _run(1, 2, 200, 64, False, seed=3, scale=0.37)
    o_ref, lse_ref = oracle.fwd(q, k, v, scale=0.37, causal=False)
    assert_close("o", o, o_ref)
    assert_close("lse", lse, lse_ref)
    q, k, v, o, lse = _run(1, 2, 200, 64, True, seed=3, scale=0.0)
    o_ref, lse_ref = oracle.fwd(q, k, v, scale=0.0, causal=True)
    assert_close("o", o, o_ref)
    assert_close("lse", lse, lse_ref)


def test_long_context_distribution_small():
    """Large logits (Q, K ~ N(0,3) with 1% of rows x8) at a size the oracle
    finishes quickly: frequent running-max rescales."""
    for d in (64, 128):
        q, k, v, o, lse = _run(1, 2, 1500, d, True, seed=4, dist="long_context")
        o_ref, lse_ref = oracle.fwd(q, k, v, causal=True)
        assert_close("o", o, o_ref)
        assert_close("lse", lse, lse_ref)


def test_deterministic_forward():
    fa = _fa()
    q, k, v, _ = inputs.qkv_do(1, 4, 700, 128, seed=1)
    q, k, v = q.to(DEV), k.to(DEV), v.to(DEV)
    o1, l1 = fa.fwd(q, k, v, causal=True)
    o2, l2 = fa.fwd(q, k, v, causal=True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
