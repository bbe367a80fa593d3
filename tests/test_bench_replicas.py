"""The multi-GPU bench path on CPU: replicas only, so the only cross-rank
steps are the barrier and the max over ranks of the elapsed time. Two gloo
ranks (127.0.0.1) report different times; both must see the slower one and
the same whole-job throughput."""
import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, "cpu")
        out[rank] = (ms, bench.replica_throughput(64, 100, world, ms))
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_time():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[0] == res[1]
    ms, value = res[0]
    assert ms == 15.0
    assert abs(value - 64 * 2 * 100 / 0.015) < 1e-6


def test_single_process_is_unchanged():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, "cpu") == 3.5
    assert bench.replica_throughput(64, 10, 1, 1.0) == 64 * 10 / 1e-3
