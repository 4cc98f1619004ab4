"""Multi-process path of bench.py on CPU: two gloo ranks, each with its own
token batch (replicas, no data-path collective); the job's throughput is all
tokens over the slowest rank's time."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms_local = [10.0, 25.0][rank]          # rank 1 is the slow one
        value, ms = bench.aggregate_throughput(32 * 100, ms_local, world, device="cpu")
        bench.barrier(world)
        q.put((rank, value, ms))
    finally:
        dist.destroy_process_group()


def test_two_rank_throughput_is_total_over_slowest():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, value, ms in res:
        assert ms == 25.0
        assert abs(value - 2 * 3200 / 0.025) < 1e-6


def test_single_rank_is_identity():
    import bench
    value, ms = bench.aggregate_throughput(3200, 20.0, 1)
    assert ms == 20.0 and abs(value - 3200 / 0.02) < 1e-9
