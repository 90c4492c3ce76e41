"""The N > 1 bench path on CPU: two gloo ranks, each timing its own replica batch,
reduce to the slowest rank's times (max over ranks), as the NCCL ranks do on GPUs."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out.put((rank, bench.slowest_rank(times[rank], "cpu")))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_report_the_slowest_times():
    world = 2
    times = [[1.0e-4, 9.0e-5, 2.0e-4, 3.0e-4], [1.5e-4, 8.0e-5, 2.5e-4, 1.0e-4]]
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, times, out)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    expect = [max(a, b) for a, b in zip(*times)]
    for r in range(world):
        assert got[r] == pytest.approx(expect, rel=0, abs=0)
