"""The benchmark's multi-rank plumbing (max over ranks, whole-job aggregate)
on CPU with two gloo ranks."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    ws, r, local = bench.dist_env()
    elapsed = 1.0 + rank  # rank 1 is the slowest
    bench.barrier()
    t_max = bench.reduce_max(elapsed)
    value = bench.aggregate(1000.0, t_max, ws)
    q.put((r, ws, t_max, value))
    dist.destroy_process_group()


def test_two_rank_max_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for r, ws, t_max, value in res:
        assert ws == 2
        assert t_max == 2.0          # max over ranks, not the local time
        assert value == 1000.0       # 2 ranks × 1000 units / 2 s


def test_single_process_identity():
    import bench
    assert bench.reduce_max(3.5) == 3.5
    assert bench.aggregate(100.0, 2.0, 1) == 50.0
