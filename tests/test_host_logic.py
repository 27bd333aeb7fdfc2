"""Host-side arithmetic pinned to the worked numbers the pages print, and the
input recipe."""
import math
import os

import numpy as np
import torch

from tiled_attention_20_b200 import inputs, perf

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [l.split() for l in f if l.strip() and not l.startswith("#")]


def test_wave_quantization_golden():
    for side, tm, tn, tiles, sms, nwaves, last in _rows("wave_quantization.txt"):
        side, tm, tn, tiles, sms, nwaves, last = map(int, (side, tm, tn, tiles, sms, nwaves, last))
        t = perf.tile_count(side, side, tm, tn)
        assert t == tiles
        assert perf.waves(t, sms) == nwaves
        assert t - (nwaves - 1) * sms == last


def test_roofline_golden():
    for flops, nbytes, bw, peak, inten, bound in _rows("roofline_example.txt"):
        flops, nbytes, bw, peak, inten, bound = map(float, (flops, nbytes, bw, peak, inten, bound))
        assert flops / nbytes == inten
        assert perf.roofline_bound(peak, bw, flops / nbytes) == bound


def test_gemm_cost_golden_and_attention_flops():
    for M, K, N, flops, nbytes in _rows("gemm_cost.txt"):
        M, K, N, flops, nbytes = map(int, (M, K, N, flops, nbytes))
        assert 2 * M * K * N == flops
        assert 2 * (M * K + K * N + M * N) == nbytes
    # attention forward = two N x N x d GEMMs per head
    B, H, N, d = 2, 32, 4096, 128
    assert perf.attention_flops(B, H, N, d, False, False) == B * H * 2 * (2 * N * d * N)
    assert perf.attention_flops(B, H, N, d, True, False) == B * H * 2 * N * d * N
    assert perf.attention_flops(B, H, N, d, True, True) == 2.5 * B * H * 2 * N * d * N


def test_inputs_seeded_and_bf16():
    a = inputs.qkv_do(1, 2, 64, 64, seed=0)
    b = inputs.qkv_do(1, 2, 64, 64, seed=0)
    c = inputs.qkv_do(1, 2, 64, 64, seed=1)
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16 and x.is_contiguous()
        assert torch.equal(x, y)
    assert not torch.equal(a[0], c[0])
    # the first draw is torch.randn(fp32) rounded to bf16
    g = torch.Generator().manual_seed(0)
    ref = torch.randn((1, 2, 64, 64), generator=g).to(torch.bfloat16)
    assert torch.equal(a[0], ref)


def test_long_context_recipe():
    N = 1000
    q, k, v, dO = inputs.qkv_do(1, 2, N, 64, seed=0, dist="long_context")
    n_big = math.ceil(0.01 * N)
    for t in (q, k):
        rms = t.float().pow(2).mean(dim=-1).sqrt()[0]  # [H, N]
        for h in range(2):
            big = (rms[h] > 12).sum().item()  # rows x8 have rms ~24, others ~3
            assert big == n_big
    assert abs(v.float().std().item() - 1.0) < 0.05
    assert abs(dO.float().std().item() - 1.0) < 0.05


def test_sweep_has_48_cases():
    ws = inputs.sweep_workloads()
    assert len(ws) == 48
    assert len({w.name for w in ws}) == 48


def test_fp8_input_recipe():
    """fp8_qkv: per (b, h) the largest |x8| is the E4M3 maximum 448, and
    x8 * descale reproduces the fp32 draws within E4M3 rounding (relative
    2^-4 for normals, absolute 2^-10 * descale below the normal range)."""
    import torch
    q8, k8, v8, fq, fk, fv = inputs.fp8_qkv(2, 3, 200, 128, seed=4)
    for x8 in (q8, k8, v8):
        assert x8.dtype == torch.float8_e4m3fn and x8.shape == (2, 3, 200, 128)
        assert torch.all(x8.float().abs().amax(dim=(2, 3)) == 448.0)
    # the same fp32 draws as the bf16 recipe (bf16 rounding of both agrees to 2^-4)
    q, k, v, _ = inputs.qkv_do(2, 3, 200, 128, seed=4)
    for x8, f, ref in ((q8, fq, q), (k8, fk, k), (v8, fv, v)):
        deq = x8.double() * f.double()[:, :, None, None]
        r = ref.double()
        tol = torch.maximum(2.0 ** -4 * r.abs() + 2.0 ** -8 * r.abs(),
                            (2.0 ** -10) * f.double()[:, :, None, None])
        assert torch.all((deq - r).abs() <= tol)


def test_decode_input_recipe():
    """decode_qkv: seeded (same seed, same tensors), bf16, and ragged lengths
    drawn in [L/2, L] (all L without ragged)."""
    import torch
    a = inputs.decode_qkv(3, 2, 4, 100, 64, seed=9, ragged=True)
    b = inputs.decode_qkv(3, 2, 4, 100, 64, seed=9, ragged=True)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    q, k, v, lens = a
    assert q.dtype == k.dtype == v.dtype == torch.bfloat16
    assert q.shape == (3, 2, 4, 64) and k.shape == v.shape == (3, 2, 100, 64)
    assert lens.dtype == torch.int32 and torch.all((lens >= 50) & (lens <= 100))
    _, _, _, full = inputs.decode_qkv(3, 2, 4, 100, 64, seed=9)
    assert torch.all(full == 100)
    for w in (inputs.DECODE_B8, inputs.DECODE_B8_RAGGED, inputs.DECODE_SPEC, inputs.DECODE_LONG):
        assert 1 <= w.Nq <= 8 and w.d in (64, 128)
