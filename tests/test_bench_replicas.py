"""Host logic of the multi-GPU bench path (replicas, no data-path
collective), on CPU with world_size-2 gloo process groups: timings reduce
to the maximum over ranks and the job rate counts every rank's tokens over
the slowest rank's time."""
import os
import socket
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [10.0 + rank, 100.0 - 7 * rank]
        got = bench.max_over_ranks(mine, dist, "cpu")
        rate = bench.replica_rate(world, 128 * 3, got[1])
        q.put((rank, got, rate))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_replica_rate_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, rate in res:
        assert got == [11.0, 100.0]  # element-wise maximum over both ranks
        assert rate == pytest.approx(2 * 128 * 3 / 0.1)


def test_single_process_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1.5, 2.5], None, "cpu") == [1.5, 2.5]
    assert bench.replica_rate(1, 128, 1000.0) == pytest.approx(128.0)
