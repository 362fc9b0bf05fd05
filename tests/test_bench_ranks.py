"""Multi-rank bench logic on CPU: two gloo ranks reduce their step times to the slowest
rank, and the whole-job value counts every rank's bytes over that time (weak scaling)."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [1.0 + rank, 5.0 - rank, 0.25 * (rank + 1), 7.0]
        got = bench.max_over_ranks(local, world, torch.device("cpu"))
        q.put((rank, got, bench.whole_job_gbs(world, 2e9, got[0])))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, got, value in res:
        assert got == [2.0, 5.0, 0.5, 7.0]                 # element-wise max over both ranks
        assert value == pytest.approx(2 * 2e9 / 2.0 / 1e9)   # both ranks' bytes / slowest time


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, 1.5], 1, torch.device("cpu")) == [3.0, 1.5]
    assert bench.whole_job_gbs(1, 1e9, 0.5) == pytest.approx(2.0)
