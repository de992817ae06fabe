"""The N>1 bench plumbing on CPU: two gloo ranks, barrier, max over ranks and
the weak-scaling arithmetic (each rank decodes its own replica; no collective
touches the data path)."""
import datetime
import multiprocessing as mp
import os
import socket

import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    bench.barrier(world)
    ms = 10.0 + 5.0 * rank           # per-rank step time; the slowest rank decides
    mx = bench.max_over_ranks(ms, world)
    value = bench.weak_scaling_value(1000, world, mx)
    bench.barrier(world)
    dist.destroy_process_group()
    q.put((rank, mx, value))


@pytest.mark.parametrize("world", [2])
def test_two_gloo_ranks_barrier_and_max(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    for pr in procs:
        pr.join(timeout=120)
    assert all(pr.exitcode == 0 for pr in procs)
    res = sorted(q.get(timeout=10) for _ in range(world))
    slowest = 10.0 + 5.0 * (world - 1)
    for rank, mx, value in res:
        assert mx == slowest
        assert value == pytest.approx(world * 1000 / (slowest / 1e3))
