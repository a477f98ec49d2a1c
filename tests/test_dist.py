"""Multi-rank host logic of bench.py on CPU: world size 2 over gloo.

Each rank decodes its own batch shard (weak scaling, no exchange on the data
path); the job's throughput is all ranks' bytes over the slowest rank's time."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        w = bench.rank_workload("opt66b", rank)
        elapsed = 1.0 + rank                        # rank 1 is the slower one
        value, t_max = bench.aggregate(w.algorithmic_bytes(), 10, elapsed, world, "cpu")
        seeds = [None] * world
        dist.all_gather_object(seeds, w.seed)
        results[rank] = (value, t_max, seeds, w.B, w.units)
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_the_batch_and_aggregate_on_the_slowest():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        results = m.dict()
        mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
        res = dict(results)
    import workloads
    w = workloads.CONFIGS["opt66b"]
    for rank in range(world):
        value, t_max, seeds, B, units = res[rank]
        assert t_max == 2.0                                   # max over ranks
        assert abs(value - world * w.algorithmic_bytes() * 10 / 2.0 / 1e9) < 1e-6
        assert len(set(seeds)) == world                       # distinct shards
        assert B == w.B and units == w.units                  # fixed work per rank


def test_single_rank_needs_no_process_group():
    import bench
    value, t_max = bench.aggregate(1e9, 5, 2.0, 1)
    assert t_max == 2.0 and value == 2.5
