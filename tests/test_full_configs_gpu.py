"""Parity at the full workload sizes, through the same calls and launch shapes
bench.py times (fa.fwd + fa.bwd with a library-sized workspace).

The fp64 oracle cannot do every head of the large workloads in test time, so
it checks whole heads sampled from each problem (all rows and gradients of
those heads); properties that hold at any size are checked on every head:
causal row 0 equals V_0 bit for bit and its lse equals scale*q_0.k_0, the
gradient sum rules (sum_j dK_j = 0, sum_j dV_j = sum_i dO_i) hold within the
kernel's rounding bounds, and the outputs are finite."""
import math

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


def _run(w):
    fa = _fa()
    q, k, v, dO = inputs.for_workload(w)
    qd, kd, vd, dOd = (t.to(DEV) for t in (q, k, v, dO))
    o, lse = fa.fwd(qd, kd, vd, causal=w.causal)
    dq, dk, dv = fa.bwd(qd, kd, vd, o, dOd, lse, causal=w.causal)
    fa.check_device_errors()
    return (q, k, v, dO), tuple(t.cpu() for t in (o, lse, dq, dk, dv))


def _check_heads(w, cpu_in, gpu_out, heads, scaled=False):
    q, k, v, dO = cpu_in
    o, lse, dq, dk, dv = gpu_out
    cmp = assert_close_scaled if scaled else assert_close
    for (b, h) in heads:
        sl = lambda t: t[b:b + 1, h:h + 1]
        o_r, lse_r = oracle.fwd(sl(q), sl(k), sl(v), causal=w.causal)
        dq_r, dk_r, dv_r, _, _ = oracle.bwd(sl(q), sl(k), sl(v), sl(dO), causal=w.causal)
        ctx = f"{w.name} head ({b},{h})"
        cmp("o", sl(o), o_r, ctx=ctx)
        assert_close("lse", sl(lse), lse_r, ctx=ctx)
        cmp("dq", sl(dq), dq_r, ctx=ctx)
        cmp("dk", sl(dk), dk_r, ctx=ctx)
        cmp("dv", sl(dv), dv_r, ctx=ctx)


def _check_all_heads_properties(w, cpu_in, gpu_out):
    q, k, v, dO = cpu_in
    o, lse, dq, dk, dv = gpu_out
    for t in (o, lse, dq, dk, dv):
        assert torch.isfinite(t.float()).all()
    if w.causal:
        assert torch.equal(o[:, :, 0], v[:, :, 0])
        s00 = (q[:, :, 0].double() * k[:, :, 0].double()).sum(-1) / math.sqrt(w.d)
        assert np.abs(np64(lse[:, :, 0]) - s00.numpy()).max() <= 1e-3 * max(1.0, float(s00.abs().max()))
    # Gradient sum rules on every head: key-shift invariance gives
    # sum_j dK_j = 0, rows of P summing to one give sum_j dV_j = sum_i dO_i.
    # Bounds from the kernel's rounding model, doubled: bf16 operands P and dS
    # (relative 2^-9), D formed from the bf16 O, and the bf16 rounding of each
    # output element (another 2^-9 relative).
    u = 2.0 ** -9
    scale = 1 / math.sqrt(w.d)
    for bi in range(w.B):  # one batch entry at a time keeps host memory small
        dk64, dv64, dO64, q64, o64 = (np64(t[bi]) for t in (dk, dv, dO, q, o))
        dd = np.abs(dO64 * o64).sum(axis=2, keepdims=True)
        bound_k = 2 * (2 * u * np.abs(dk64).sum(axis=1)
                       + scale * u * (dd * np.abs(q64)).sum(axis=1)) + 1e-6
        err_k = np.abs(dk64.sum(axis=1))
        assert (err_k <= bound_k).all(), f"sum dK: {err_k.max():.3e} (batch {bi})"
        bound_v = 2 * u * (np.abs(dO64).sum(axis=1) + np.abs(dv64).sum(axis=1)) + 1e-6
        assert (np.abs(dv64.sum(axis=1) - dO64.sum(axis=1)) <= bound_v).all(), \
            f"sum dV != sum dO (batch {bi})"


def test_gpt_causal_workload():
    """B=2, H=32, N=4096, d=128, causal: the benchmark workload."""
    w = inputs.GPT_CAUSAL
    cpu_in, gpu_out = _run(w)
    _check_all_heads_properties(w, cpu_in, gpu_out)
    _check_heads(w, cpu_in, gpu_out, [(0, 0), (1, 31), (0, 17)])


def test_long_context_workload():
    """B=1, H=16, N=16384, d=128, causal, Q,K ~ N(0,3) with 1% of rows x8.
    Logits reach the hundreds and gradients are far from unit scale, so the
    bound on O and the gradients is scaled by the result's magnitude."""
    w = inputs.LONG_CONTEXT
    cpu_in, gpu_out = _run(w)
    _check_all_heads_properties(w, cpu_in, gpu_out)
    _check_heads(w, cpu_in, gpu_out, [(0, 5)], scaled=True)


@pytest.mark.parametrize("w", [inputs.MID_NC, inputs.MID_C], ids=lambda w: w.name)
def test_mid_workloads_every_head(w):
    """B=4, H=16, N=1024, d=64, both masks: every head against the oracle."""
    cpu_in, gpu_out = _run(w)
    _check_all_heads_properties(w, cpu_in, gpu_out)
    q, k, v, dO = cpu_in
    o, lse, dq, dk, dv = gpu_out
    o_r, lse_r = oracle.fwd(q, k, v, causal=w.causal)
    dq_r, dk_r, dv_r, _, _ = oracle.bwd(q, k, v, dO, causal=w.causal)
    for name, a, r in (("o", o, o_r), ("lse", lse, lse_r), ("dq", dq, dq_r), ("dk", dk, dk_r),
                       ("dv", dv, dv_r)):
        assert_close(name, a, r, ctx=w.name)


@pytest.mark.parametrize("w", inputs.sweep_workloads(), ids=lambda w: w.name)
def test_boundary_wave_sweep(w):
    """H=16, d in {64,128}, B in {1,8}, N in {1792,1793,2048,2049,4000,8192},
    both masks, forward and backward: ragged tails, masking and wave counts
    on 148 SMs.  One head is checked against the oracle (the last head, whose
    rows sit at the end of every buffer), all heads for properties."""
    cpu_in, gpu_out = _run(w)
    _check_all_heads_properties(w, cpu_in, gpu_out)
    _check_heads(w, cpu_in, gpu_out, [(w.B - 1, w.H - 1)])
