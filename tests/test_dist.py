"""Rank logic of N-GPU runs, exercised as world-size-2 gloo process groups on the CPU."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from ternary_weight_linear_03_b200 import dist as bldist


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        r, w, lr = bldist.rank_env()
        slowest = bldist.max_over_ranks(1.5 + rank, dist)
        dist.barrier()
        results[rank] = (r, w, lr, slowest, bldist.seed_offset(r), bldist.row_shard(10, w, r))
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_logic():
    world = 2
    manager = mp.get_context("spawn").Manager()
    results = manager.dict()
    mp.spawn(_worker, args=(world, _free_port(), results), nprocs=world, join=True)
    assert set(results.keys()) == {0, 1}
    for rank in range(world):
        r, w, lr, slowest, off, shard = results[rank]
        assert (r, w, lr) == (rank, world, rank)
        assert slowest == 2.5  # max over ranks
    assert results[0][4] != results[1][4]  # replicas get different seeds
    assert results[0][5] == (0, 5) and results[1][5] == (5, 10)


@pytest.mark.parametrize("N,world", [(10, 3), (28672, 8), (1, 4), (4096, 1)])
def test_row_shards_tile_the_rows(N, world):
    shards = [bldist.row_shard(N, world, r) for r in range(world)]
    assert shards[0][0] == 0 and shards[-1][1] == N
    for (a0, a1), (b0, b1) in zip(shards, shards[1:]):
        assert a1 == b0
    sizes = [b - a for a, b in shards]
    assert max(sizes) - min(sizes) <= 1


def test_max_over_ranks_without_group():
    assert bldist.max_over_ranks(3.0) == 3.0
