"""The multi-GPU host path with two ranks over gloo on CPU.

Each rank owns a round-robin shard of the sequences and runs its own step;
the job's time is the slowest rank's and its keys are the sum over ranks.
This exercises the same reductions ``bench.py`` performs under torchrun,
without a GPU.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from rope_aware_kv_tri_b200.sharding import (check_partition, freed_consistent, keys_per_second, reduce_job,
                                             shard_heads, shard_seed, shard_sequences)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, S, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = shard_sequences(S, world, rank)
        # a stand-in for the rank's timed steps: rank r is slower by r ms
        ms = 10.0 + rank
        keys = 1000 * len(mine)
        freed = 7 * len(mine)
        gathered = [None] * world
        dist.all_gather_object(gathered, mine)
        t, k, f = reduce_job(dist, ms, keys, freed)
        out[rank] = (gathered, t, k, f, shard_seed(0, rank))
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_and_reduce():
    world, S = 2, 5
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, S, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    r0, r1 = out[0], out[1]
    shards = r0[0]
    assert shards == r1[0] and check_partition(shards, S)
    assert shards == [[0, 2, 4], [1, 3]]
    assert r0[1] == r1[1] == 11.0                  # max over ranks
    assert r0[2] == r1[2] == 5000 and r0[3] == r1[3] == 35
    assert r0[4] != r1[4]                          # independent caches
    assert keys_per_second(r0[2], 3, r0[1]) == pytest.approx(5000 * 3 / 0.011)


def test_single_process_reduction_and_errors():
    assert reduce_job(None, 2.5, 10, 3) == (2.5, 10, 3)
    assert shard_sequences(3, 1, 0) == [0, 1, 2]
    with pytest.raises(ValueError):
        shard_sequences(3, 2, 2)
    with pytest.raises(ValueError):
        keys_per_second(10, 1, 0.0)
    assert not check_partition([[0, 1], [1]], 2)


def _heads_worker(rank, world, port, out, freed_by_rank):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = shard_heads(8, world, rank)
        gathered = [None] * world
        dist.all_gather_object(gathered, mine)
        same = freed_consistent(dist, freed_by_rank[rank])
        t, k, f = reduce_job(dist, 5.0 + rank, 100 * len(mine), freed_by_rank[rank])
        out[rank] = (gathered, same, t, k, f)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("freed_by_rank,consistent", [((30, 30), True), ((30, 29), False)])
def test_two_ranks_head_sharding_and_freed_all_reduce(freed_by_rank, consistent):
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_heads_worker, args=(r, world, port, out, freed_by_rank)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    heads = out[0][0]
    assert heads == out[1][0] == [[0, 1, 2, 3], [4, 5, 6, 7]]
    assert out[0][1] is consistent and out[1][1] is consistent
    assert out[0][2] == out[1][2] == 6.0
    assert out[0][3] == 800 and out[0][4] == sum(freed_by_rank)


def test_head_sharding_rules():
    assert shard_heads(8, 1, 0) == list(range(8))
    assert shard_heads(8, 8, 3) == [3]
    with pytest.raises(ValueError):
        shard_heads(8, 3, 0)
    assert freed_consistent(None, 5)
