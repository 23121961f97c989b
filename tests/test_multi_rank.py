"""The N > 1 path of bench.py on CPU: world-size-2 gloo ranks run independent
replicas, time is the maximum over ranks, and the job's throughput counts
every rank's tokens (weak scaling).  No GPU and no data-path collective."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, times, out):
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        t = bench.max_over_ranks(times[rank], torch.device("cpu"), world)
        e = bench.max_over_ranks(times[rank] * 2.0, torch.device("cpu"), world)
        out[rank] = (t, e, bench.job_tokens_per_s(world, 4, 128, t))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    times = [3.25, 4.5]
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, port, times, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        t, e, v = res[r]
        assert t == max(times)
        assert e == 2.0 * max(times)
        assert v == pytest.approx(world * 4 * 128 / (max(times) / 1e3))


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(1.5, torch.device("cpu"), 1) == 1.5
    assert bench.job_tokens_per_s(1, 4, 10, 2.0) == pytest.approx(20000.0)
