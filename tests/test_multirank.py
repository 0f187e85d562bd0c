"""The multi-GPU host path of bench.py on CPU: two gloo ranks check the head
sharding (weak scaling, no data-path collective) and the max-over-ranks timing
that turns per-rank times into whole-job throughput."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        start, stop = bench.shard_heads(32, world, rank)
        # every rank reports its shard; all-gather them to check the cover
        shard = torch.tensor([start, stop], dtype=torch.int64)
        shards = [torch.zeros(2, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(shards, shard)
        my_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
        slowest = bench.max_over_ranks(my_ms)
        value = bench.job_throughput(1e12, 4, world, slowest)
        out[rank] = (shards, slowest, value)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        shards, slowest, value = res[rank]
        covered = sorted(h for s in shards for h in range(int(s[0]), int(s[1])))
        assert covered == list(range(32 * world))       # each head exactly once
        assert slowest == 15.0                           # max over ranks
        assert value == pytest.approx(1e12 * 4 * world / 15e-3 / 1e12)
