"""GEMM parity on the GPU: fa_gemm through the C ABI against the fp64 oracle
(same seeded bf16 inputs), over sizes of every divisibility class (1, 2, 8,
16, 32), ragged tile edges, the wave boundaries of 148 SMs, strided operands
and an unaligned base pointer.

Tolerance: products of bf16 values are exact in fp32, so the error is the
fp32 accumulation, at most 2 K 2^-24 (|A| |B|)_ij, plus the bf16 rounding of
C, at most 2^-9 |C_ij| (bounds doubled for margin)."""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import np64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _fa():
    import tiled_attention_20_b200.fa as fa
    return fa


def _mats(M, N, K, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    a = torch.randn((M, K), generator=g).to(torch.bfloat16)
    b = torch.randn((K, N), generator=g).to(torch.bfloat16)
    return a, b


def _check(c_gpu, a, b, ctx=""):
    ref = oracle.gemm(a, b)
    K = a.shape[1]
    bound = 2 * (2 * K * 2.0 ** -24 * (np.abs(np64(a)) @ np.abs(np64(b))) + 2.0 ** -9 * np.abs(ref)) + 1e-6
    err = np.abs(np64(c_gpu) - ref)
    assert np.isfinite(np64(c_gpu)).all(), ctx
    worst = float((err / bound).max())
    assert worst <= 1.0, f"C error exceeds the bound by {worst:.2f}x {ctx}"


@pytest.mark.parametrize("n", [1, 2, 7, 8, 15, 16, 31, 32, 63, 64, 65, 127, 128, 129, 255, 256,
                               257, 300, 1000])
def test_square_sizes(n):
    a, b = _mats(n, n, n, seed=n)
    c = _fa().gemm(a.to(DEV), b.to(DEV))
    _fa().check_device_errors()
    _check(c.cpu(), a, b, f"n={n}")


@pytest.mark.parametrize("M,N,K", [(1, 128, 64), (256, 1, 64), (256, 128, 1), (17, 300, 129),
                                   (513, 130, 70), (1792, 1792, 64), (1793, 1793, 64),
                                   (2304, 2304, 256), (4096, 256, 4096), (300, 4100, 33),
                                   (3333, 3400, 100), (4096, 4100, 72), (4100, 4096, 1)])
def test_rectangular_and_wave_edges(M, N, K):
    """Ragged edges in both tilings (256 x 256 is used from 148 wide tiles up)."""
    a, b = _mats(M, N, K, seed=M + N + K)
    c = _fa().gemm(a.to(DEV), b.to(DEV))
    _fa().check_device_errors()
    _check(c.cpu(), a, b, f"{M}x{N}x{K}")


def test_strided_operands_and_output():
    """Row strides larger than the width (aligned and unaligned) and a padded C."""
    fa = _fa()
    a, b = _mats(300, 200, 150, seed=5)
    ap = torch.zeros((300, 157), dtype=torch.bfloat16)   # lda = 157: not a multiple of 8
    ap[:, :150] = a
    bp = torch.zeros((150, 208), dtype=torch.bfloat16)   # ldb = 208: aligned
    bp[:, :200] = b
    cp = torch.full((300, 211), 7.0, dtype=torch.bfloat16, device=DEV)  # ldc = 211
    fa.gemm(ap.to(DEV)[:, :150], bp.to(DEV)[:, :200], out=cp[:, :200])
    fa.check_device_errors()
    _check(cp[:, :200].cpu(), a, b, "strided")
    assert torch.all(cp[:, 200:] == 7.0), "columns past N were written"


def test_unaligned_base_pointer():
    """An operand starting 2 bytes past a 16-byte boundary goes through the
    aligned copy."""
    fa = _fa()
    a, b = _mats(100, 96, 64, seed=6)
    buf = torch.zeros(100 * 64 + 1, dtype=torch.bfloat16, device=DEV)
    a_view = buf[1:].view(100, 64)
    a_view.copy_(a.to(DEV))
    c = fa.gemm(a_view, b.to(DEV))
    fa.check_device_errors()
    _check(c.cpu(), a, b, "unaligned base")
