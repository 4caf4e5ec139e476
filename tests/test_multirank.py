"""Multi-rank host logic of the benchmark on CPU (gloo, two ranks).

The replicated path has no data-path collective: each rank runs its own
layer, and only the timing and the work are combined, as the slowest rank's
time and the sum of all ranks' work."""
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


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    t, w = bench.aggregate_over_ranks(1.5 + rank, 10.0 * (rank + 1), world, "cpu")
    out.put((rank, t, w))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_aggregation():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(out.get(timeout=10) for _ in range(world))
    for rank, t, w in res:
        assert t == 2.5          # the slowest rank's time, on every rank
        assert w == 30.0         # the work of both ranks


def test_single_rank_passthrough():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.aggregate_over_ranks(0.25, 7.0, 1, "cpu") == (0.25, 7.0)
