"""Host-side performance arithmetic: FLOP convention, tile and wave counts,
and the roofline bound.  No attention numerics live here.
"""
from __future__ import annotations

import math


def attention_flops(B: int, H: int, N: int, d: int, causal: bool, backward: bool) -> float:
    """Algorithmic FLOPs of one pass.

    Forward: two GEMMs of 2*N*N*d each per head (S = Q K^T and O = P V; a GEMM
    of M x K by K x N costs about 2MKN, "第17讲 Tensor Core、HBM、SRAM 与
    FlashAttention", §5.3), i.e. 4*B*H*N^2*d, halved when causal.  Backward:
    2.5 x the forward (five GEMMs instead of two).
    """
    f = 4.0 * B * H * N * N * d
    if causal:
        f *= 0.5
    return 2.5 * f if backward else f


def attention_bytes(B: int, H: int, N: int, d: int, backward: bool, elem: int = 2) -> float:
    """Algorithmic HBM bytes of one pass (each operand read once, each result
    written once).  Forward: Q, K, V read, O written, lse (fp32) written.
    Backward: Q, K, V, O, dO read, dQ, dK, dV written; lse read, D written."""
    per_head = (8 if backward else 4) * N * d * elem + (8 if backward else 4) * N
    return float(B * H * per_head)


def tile_count(M: int, N: int, tile_m: int, tile_n: int) -> int:
    """Output tiles of an M x N result cut into tile_m x tile_n blocks."""
    return math.ceil(M / tile_m) * math.ceil(N / tile_n)


def waves(tiles: int, sms: int) -> int:
    """Full or partial waves needed when every SM runs one tile at a time."""
    return math.ceil(tiles / sms)


def roofline_bound(peak_flops: float, bandwidth: float, intensity: float) -> float:
    """Attainable performance P <= min(P_peak, BW * I) (same page, §6.2)."""
    return min(peak_flops, bandwidth * intensity)
