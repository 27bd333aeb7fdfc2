"""Seeded synthetic inputs shared by the oracle tests, the GPU parity tests and
the benchmark.

This module holds no attention arithmetic: only random draws, the workload
shapes, and bf16 rounding of the draws.  Draws happen on the CPU with a
``torch.Generator`` so that both sides see bit-identical inputs.

Recipe (one generator per call, seeded with ``seed``):

1. ``torch.randn`` in fp32, in the order Q, K, V, dO, each [B, H, N, d].
2. ``dist == "long_context"`` (the long-context workload): Q and K are scaled
   by 3 (standard deviation 3), then, for each (b, h) in order, ceil(0.01 N)
   query rows and then ceil(0.01 N) key rows, drawn without replacement with
   ``torch.randperm`` from the same generator, are multiplied by 8.  V and dO
   keep standard deviation 1.
3. Everything is rounded to bf16 (round to nearest even).

FP8 inputs (``fp8_qkv``): the fp32 draws of steps 1-2 (before any bf16
rounding), then per (b, h) and per tensor a dequantisation factor
amax / 448 (448 is the largest E4M3 value; 1 for an all-zero head) and the
E4M3 value of x / factor (``torch.float8_e4m3fn``, round to nearest even).

Decode inputs (``decode_qkv``): one generator per call; ``torch.randn`` fp32
for q [B, H, Nq, d], then the caches k, v [B, H, L, d]; with ``ragged`` the
per-batch valid lengths are then drawn uniformly from [L/2, L] with
``torch.randint`` (else every batch has L rows); bf16 rounding last.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    """One attention problem: shape, mask, which passes, value distribution."""
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    backward: bool
    dist: str = "normal"
    seed: int = 0


# The five workload families the method is measured and checked on.
SMALL_FWD = Workload("fwd_nc_B1_H2_N256_d64", 1, 2, 256, 64, False, False)
MID_NC = Workload("fwdbwd_nc_B4_H16_N1024_d64", 4, 16, 1024, 64, False, True)
MID_C = Workload("fwdbwd_c_B4_H16_N1024_d64", 4, 16, 1024, 64, True, True)
GPT_CAUSAL = Workload("fwdbwd_c_B2_H32_N4096_d128", 2, 32, 4096, 128, True, True)
LONG_CONTEXT = Workload("fwdbwd_c_B1_H16_N16384_d128_lc", 1, 16, 16384, 128, True, True,
                        dist="long_context")


@dataclass(frozen=True)
class DecodeWorkload:
    """A decode step: Nq new queries per head against an L-row cache."""
    name: str
    B: int
    H: int
    Nq: int
    L: int
    d: int
    causal: bool
    ragged: bool = False
    seed: int = 0


# Decode-shaped calls: GPT-style heads (H=32, d=128) at batch 8 reading an
# 8192-token cache (1 GiB of K and V, well above L2), its ragged-length and
# speculative (Nq=4, causal) variants, and a small-batch long-cache case.
DECODE_B8 = DecodeWorkload("decode_B8_H32_Nq1_L8192_d128", 8, 32, 1, 8192, 128, False)
DECODE_B8_RAGGED = DecodeWorkload("decode_B8_H32_Nq1_L8192_d128_ragged", 8, 32, 1, 8192, 128,
                                  False, ragged=True)
DECODE_SPEC = DecodeWorkload("decode_B8_H32_Nq4_L8192_d128_causal", 8, 32, 4, 8192, 128, True)
DECODE_LONG = DecodeWorkload("decode_B1_H32_Nq1_L65536_d128", 1, 32, 1, 65536, 128, False)


def decode_qkv(B: int, H: int, Nq: int, L: int, d: int, seed: int = 0, ragged: bool = False):
    """(q, k_cache, v_cache, lens): bf16 [B,H,Nq,d], [B,H,L,d], [B,H,L,d] and
    int32 [B] valid lengths."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    q = torch.randn((B, H, Nq, d), generator=g, dtype=torch.float32)
    k = torch.randn((B, H, L, d), generator=g, dtype=torch.float32)
    v = torch.randn((B, H, L, d), generator=g, dtype=torch.float32)
    if ragged:
        lens = torch.randint(L // 2, L + 1, (B,), generator=g, dtype=torch.int32)
    else:
        lens = torch.full((B,), L, dtype=torch.int32)
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16), lens


def sweep_workloads():
    """The boundary / wave sweep: H=16, d in {64,128}, B in {1,8},
    N in {1792,1793,2048,2049,4000,8192}, causal and not; fwd and bwd."""
    out = []
    for d in (64, 128):
        for B in (1, 8):
            for N in (1792, 1793, 2048, 2049, 4000, 8192):
                for causal in (False, True):
                    tag = "c" if causal else "nc"
                    out.append(Workload(f"sweep_{tag}_B{B}_H16_N{N}_d{d}", B, 16, N, d,
                                        causal, True))
    return out


def fp8_qkv(B: int, H: int, N: int, d: int, seed: int = 0, dist: str = "normal"):
    """(q8, k8, v8, descale_q, descale_k, descale_v): float8_e4m3fn
    [B, H, N, d] tensors and fp32 [B, H] factors with x ~ x8 * factor."""
    q, k, v, _ = _draw_fp32(B, H, N, d, seed, dist)
    out8, scales = [], []
    for x in (q, k, v):
        amax = x.abs().amax(dim=(2, 3))
        f = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax)).to(torch.float32)
        out8.append((x / f[:, :, None, None]).to(torch.float8_e4m3fn).contiguous())
        scales.append(f.contiguous())
    return (*out8, *scales)


def qkv_do(B: int, H: int, N: int, d: int, seed: int = 0, dist: str = "normal",
           device: str | torch.device = "cpu"):
    """(q, k, v, dO) as contiguous bf16 [B, H, N, d] tensors."""
    q, k, v, dO = _draw_fp32(B, H, N, d, seed, dist)
    return tuple(t.to(torch.bfloat16).contiguous().to(device) for t in (q, k, v, dO))


def _draw_fp32(B: int, H: int, N: int, d: int, seed: int, dist: str):
    """Steps 1-2 of the recipe: the fp32 draws before rounding."""
    g = torch.Generator(device="cpu").manual_seed(int(seed))
    shape = (B, H, N, d)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    dO = torch.randn(shape, generator=g, dtype=torch.float32)
    if dist == "long_context":
        q.mul_(3.0)
        k.mul_(3.0)
        n_big = math.ceil(0.01 * N)
        for b in range(B):
            for h in range(H):
                iq = torch.randperm(N, generator=g)[:n_big]
                ik = torch.randperm(N, generator=g)[:n_big]
                q[b, h, iq] *= 8.0
                k[b, h, ik] *= 8.0
    elif dist != "normal":
        raise ValueError(f"unknown distribution {dist!r}")
    return q, k, v, dO


def for_workload(w: Workload, device="cpu"):
    return qkv_do(w.B, w.H, w.N, w.d, seed=w.seed, dist=w.dist, device=device)
