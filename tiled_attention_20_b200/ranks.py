"""Host-side plumbing for running the attention path on several GPUs of one
node, one process per GPU.

Every (b, h) head is independent in the forward and the backward, so ranks
share no data: each rank runs its own problem (weak scaling) and the only
communication is timing bookkeeping — a barrier around the timed region and
the maximum of the per-rank step times.
"""
from __future__ import annotations

import os
from dataclasses import dataclass


@dataclass(frozen=True)
class RankInfo:
    rank: int
    world: int
    local_rank: int


def rank_info(env=None) -> RankInfo:
    """RANK / WORLD_SIZE / LOCAL_RANK as torchrun sets them (1 process if unset)."""
    env = os.environ if env is None else env
    return RankInfo(int(env.get("RANK", "0")), int(env.get("WORLD_SIZE", "1")),
                    int(env.get("LOCAL_RANK", "0")))


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own synthetic inputs."""
    return base_seed + rank


def shard_heads(n_heads: int, rank: int, world: int) -> range:
    """Contiguous block of head indices owned by `rank` when a fixed set of
    n_heads heads is split across `world` ranks (sizes differ by at most 1)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    base, extra = divmod(n_heads, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """Maximum of `value` over all ranks (the slowest rank sets the step time)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_rate(flops_per_rank: float, world: int, step_ms: float) -> float:
    """Whole-job FLOP/s: all ranks' work over the slowest rank's step time."""
    return flops_per_rank * world / (step_ms * 1e-3)
