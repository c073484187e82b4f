"""Multi-rank logic of the benchmark on CPU: world size 2 over gloo (127.0.0.1).

Each rank decodes its own batch (weak scaling, no data-path collective); the job's time is the
max over ranks and its throughput counts every rank's tokens."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    mine = bench.shard_requests(64, rank, world)
    got = [None] * world
    dist.all_gather_object(got, mine)
    ms = 10.0 + 5.0 * rank                      # rank 1 is slower
    value, mx = bench.job_throughput(64, ms, world, torch.device("cpu"))
    q.put((rank, got, value, mx))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_sharding_and_max_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, shards, value, mx in res:
        flat = sorted(x for s in shards for x in s)
        assert flat == list(range(128))                       # disjoint and complete
        assert not set(shards[0]) & set(shards[1])
        assert mx == 15.0                                     # slowest rank
        assert abs(value - 128 / 15e-3) < 1e-6                # all ranks' tokens / max time
