"""The benchmark's multi-process path on CPU: two gloo ranks, the same helpers
bench.py uses under torchrun (process-group setup, barrier, max over ranks,
whole-job aggregation).  The step itself has no data-path exchange; N ranks are
N independent replicas."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist

    r, w, _ = bench.dist_setup(world, backend="gloo")
    assert (r, w) == (rank, world)
    bench.barrier(w, cuda=False)
    slowest = bench.reduce_max(0.05 + 0.01 * rank, w, device="cpu")   # ms per step of this replica
    value = bench.whole_job_gbs(30_000_000, slowest, w)
    bench.barrier(w, cuda=False)
    dist.destroy_process_group()
    out.put((rank, slowest, value))


def test_two_gloo_ranks_take_the_slowest_replica():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, slowest, value in got:
        assert slowest == pytest.approx(0.06)
        assert value == pytest.approx(2 * 30_000_000 / 0.06e-3 / 1e9)


def test_whole_job_rate_single_rank():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.whole_job_gbs(1e9, 1000.0, 1) == pytest.approx(1.0)
    assert bench.reduce_max(3.5, 1) == 3.5
