"""Decode parity on the GPU: fa_decode through the C ABI against the fp64
oracle's decode (same seeded bf16 inputs), over query counts, cache lengths
and strides, per-batch lengths, the causal mask, forced and automatic
splits, empty rows, and the full-size decode workloads on sampled heads."""
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


def _decode(q, k, v, lens=None, causal=False, num_splits=0, nk=None, scale=None):
    fa = _fa()
    lens_d = None if lens is None else lens.to(DEV)
    o, lse = fa.decode(q.to(DEV), k.to(DEV), v.to(DEV), cache_lens=lens_d, causal=causal,
                       num_splits=num_splits, nk=nk, scale=scale)
    fa.check_device_errors()
    return o, lse


def _check(o, lse, q, k, v, lens=None, causal=False, scale=None, ctx=""):
    """O within the forward's tolerance; lse within 1e-3 where finite and
    -inf exactly where the oracle has no visible key."""
    o_ref, lse_ref = oracle.decode(q, k, v, scale=scale, causal=causal,
                                   lens=None if lens is None else lens.numpy())
    assert_close("o", o, o_ref, ctx=ctx)
    lg, lr = np64(lse), lse_ref
    empty = np.isneginf(lr)
    assert np.array_equal(np.isneginf(lg), empty), f"lse -inf pattern differs {ctx}"
    if (~empty).any():
        err = float(np.abs(lg[~empty] - lr[~empty]).max())
        assert err <= 1e-3, f"lse: max err {err:.3e} {ctx}"
    assert np.all(np64(o)[empty] == 0.0), f"rows with no key must be 0 {ctx}"


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Nq", [1, 2, 3, 4, 5, 8])
@pytest.mark.parametrize("causal", [False, True])
def test_query_counts(Nq, d, causal):
    B, H, L = 2, 3, 1000
    q, k, v, _ = inputs.decode_qkv(B, H, Nq, L, d, seed=Nq)
    o, lse = _decode(q, k, v, causal=causal)
    _check(o, lse, q, k, v, causal=causal, ctx=f"Nq={Nq} d={d} causal={causal}")


@pytest.mark.parametrize("L", [1, 2, 63, 64, 65, 127, 129, 511, 4097, 8191])
@pytest.mark.parametrize("d", [64, 128])
def test_cache_lengths(L, d):
    q, k, v, _ = inputs.decode_qkv(1, 4, 1, L, d, seed=L)
    o, lse = _decode(q, k, v)
    _check(o, lse, q, k, v, ctx=f"L={L} d={d}")


@pytest.mark.parametrize("num_splits", [1, 2, 3, 7, 16, 64])
@pytest.mark.parametrize("Nq,causal", [(1, False), (4, True)])
def test_forced_splits(num_splits, Nq, causal):
    """Every split count merges to the same answer (chunks of whole tiles,
    a ragged last chunk, chunks past the end of the cache)."""
    q, k, v, _ = inputs.decode_qkv(2, 2, Nq, 3000, 128, seed=5)
    o, lse = _decode(q, k, v, causal=causal, num_splits=num_splits)
    _check(o, lse, q, k, v, causal=causal, ctx=f"splits={num_splits}")


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("num_splits", [0, 1, 5])
def test_per_batch_lengths(causal, num_splits):
    """Ragged valid lengths, including 0 and lengths below Nq (empty causal
    rows), with NaN in every row past a batch's length: nothing past the
    length may reach the result."""
    B, H, Nq, L, d = 6, 2, 4, 700, 64
    q, k, v, _ = inputs.decode_qkv(B, H, Nq, L, d, seed=11)
    lens = torch.tensor([700, 0, 1, 3, 64, 513], dtype=torch.int32)
    kn, vn = k.clone(), v.clone()
    for b, n in enumerate(lens.tolist()):
        kn[b, :, n:] = float("nan")
        vn[b, :, n:] = float("nan")
    o, lse = _decode(q, kn, vn, lens=lens, causal=causal, num_splits=num_splits)
    _check(o, lse, q, k, v, lens=lens, causal=causal, ctx=f"causal={causal} splits={num_splits}")


def test_cache_capacity_stride():
    """ld_kv > Nk: the cache holds 1500 rows per head, 1200 are valid."""
    fa = _fa()
    q, k, v, _ = inputs.decode_qkv(2, 2, 2, 1500, 128, seed=3)
    o, lse = fa.decode(q.to(DEV), k.to(DEV), v.to(DEV), nk=1200)
    fa.check_device_errors()
    _check(o, lse, q, k[:, :, :1200], v[:, :, :1200])


@pytest.mark.parametrize("scale", [0.0, 0.02, 0.5])
def test_scales(scale):
    q, k, v, _ = inputs.decode_qkv(1, 2, 3, 900, 64, seed=4)
    o, lse = _decode(q, k, v, causal=True, scale=scale)
    _check(o, lse, q, k, v, causal=True, scale=scale, ctx=f"scale={scale}")


def test_deterministic_and_workspace_reuse():
    """Two calls on one workspace give bit-identical results (fixed merge
    order) and leave the per-head counters at zero."""
    fa = _fa()
    q, k, v, lens = inputs.decode_qkv(4, 8, 1, 5000, 128, seed=8, ragged=True)
    q, k, v, lens = q.to(DEV), k.to(DEV), v.to(DEV), lens.to(DEV)
    ws = torch.zeros(max(fa.decode_workspace_size(4, 8, 1, 5000, 128, 6), 16),
                     dtype=torch.uint8, device=DEV)
    o1, l1 = fa.decode(q, k, v, cache_lens=lens, num_splits=6, workspace=ws)
    o2, l2 = fa.decode(q, k, v, cache_lens=lens, num_splits=6, workspace=ws)
    fa.check_device_errors()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert int(ws[: 4 * 8 * 4].view(torch.int32).abs().sum()) == 0


@pytest.mark.parametrize("w", [inputs.DECODE_B8, inputs.DECODE_B8_RAGGED, inputs.DECODE_SPEC,
                               inputs.DECODE_LONG], ids=lambda w: w.name)
def test_full_size_decode_workloads(w):
    """The decode workloads at full size, in the automatic split the bench
    times; the oracle checks a sample of heads (every batch's first head and
    the last head overall)."""
    q, k, v, lens = inputs.decode_qkv(w.B, w.H, w.Nq, w.L, w.d, seed=w.seed, ragged=w.ragged)
    o, lse = _decode(q, k, v, lens=lens if w.ragged else None, causal=w.causal)
    for b in range(w.B):
        for h in sorted({0, w.H - 1} if b == w.B - 1 else {0}):
            sl = (slice(b, b + 1), slice(h, h + 1))
            _check(o[sl].cpu(), lse[sl].cpu(), q[sl], k[sl], v[sl],
                   lens=lens[b:b + 1] if w.ragged else None, causal=w.causal,
                   ctx=f"{w.name} b={b} h={h}")
