"""The multi-rank host path on CPU: two gloo ranks on 127.0.0.1 exchange their
step times the way bench.py does on GPUs (barrier, max over ranks), and the
head sharding / seeding helpers are checked."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from tiled_attention_20_b200 import ranks


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        info = ranks.rank_info()
        assert (info.rank, info.world, info.local_rank) == (rank, world, rank)
        dist.barrier()
        my_ms = 1.0 + 0.5 * rank          # rank 1 is the slow one
        worst = ranks.max_over_ranks(my_ms, dist)
        owned = list(ranks.shard_heads(64, rank, world))
        out[rank] = (worst, ranks.rank_seed(0, rank), owned[0], owned[-1], len(owned))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_step():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert res[0][0] == res[1][0] == 1.5
    assert res[0][1] != res[1][1]
    assert (res[0][2], res[0][3], res[0][4]) == (0, 31, 32)
    assert (res[1][2], res[1][3], res[1][4]) == (32, 63, 32)


def test_shard_heads_covers_all_once():
    for n in (1, 7, 64, 100):
        for world in (1, 2, 3, 8):
            got = [h for r in range(world) for h in ranks.shard_heads(n, r, world)]
            assert got == list(range(n))
    with pytest.raises(ValueError):
        ranks.shard_heads(4, 2, 2)


def test_weak_scaling_rate_and_single_process_max():
    assert ranks.weak_scaling_rate(1e12, 4, 2.0) == 2e15
    assert ranks.max_over_ranks(3.25) == 3.25
