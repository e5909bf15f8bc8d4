"""Multi-rank host logic on CPU (gloo, world size 2): shard ownership and the
max-over-ranks timing reduction used by bench.py under torchrun."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from resolution_block_sparse_b200.sharding import max_over_ranks, shard_range, weak_scaling_seed


@pytest.mark.parametrize("units,world", [(24, 2), (25, 2), (16, 8), (3, 4), (0, 2), (1, 1)])
def test_shards_cover_every_unit_once(units, world):
    owned = []
    sizes = []
    for r in range(world):
        a, b = shard_range(units, world, r)
        owned.extend(range(a, b))
        sizes.append(b - a)
    assert owned == list(range(units))
    assert max(sizes) - min(sizes) <= 1


def test_bad_shard_arguments():
    with pytest.raises(ValueError):
        shard_range(4, 0, 0)
    with pytest.raises(ValueError):
        shard_range(4, 2, 2)


def test_weak_scaling_seeds_distinct():
    seeds = {weak_scaling_seed(1004, r) for r in range(8)}
    assert len(seeds) == 8


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, results):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank "measures" a different time; everyone must see the max
        mine = [1.0 + rank, 10.0 - rank]
        got = max_over_ranks(mine)
        a, b = shard_range(24, world, rank)
        results[rank] = (got, (a, b))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    world = 2
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    results = manager.dict()
    mp.start_processes(_worker, args=(world, port, results), nprocs=world, join=True,
                       start_method="spawn")
    assert results[0][0] == [2.0, 10.0]
    assert results[1][0] == [2.0, 10.0]
    assert results[0][1] == (0, 12) and results[1][1] == (12, 24)
