"""The multi-rank path of bench.py on CPU: two gloo ranks, each timing its own
replica; the job's time is the slowest rank's and the value counts every
rank's tokens."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench

        ms = [120.0, 150.0][rank]  # rank 1 is the slow replica
        m = bench.max_over_ranks(ms, "cpu")
        v = bench.job_throughput(1000, 10, world, m)
        out[rank] = (m, v)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0] == out[1]
    m, v = out[0]
    assert m == 150.0
    assert abs(v - 2 * 1000 * 10 / 0.150) < 1e-6


def test_single_process_needs_no_group():
    import bench

    assert bench.max_over_ranks(3.5, "cpu") == 3.5
    assert bench.job_throughput(16384, 20, 1, 740.0) == 16384 * 20 / 0.74
