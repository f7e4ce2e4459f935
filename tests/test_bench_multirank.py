"""The multi-GPU bench path on CPU: two gloo ranks agree on the slowest rank's time and
the whole-job throughput (each rank is an independent replica; no data exchange)."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys

    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench

    t = bench.reduce_max(100.0 + 7.0 * rank, torch.device("cpu"))
    out.put((rank, t, bench.dist_setup(), bench.job_throughput(world, 1e12, t, 10)))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, (w, r, lr), value in res:
        assert t == 107.0 and w == 2 and r == rank == lr
        assert value == pytest.approx(2 * 1e12 / (107.0 / 10 * 1e-3) / 1e12)


def test_single_process_reduce_is_identity():
    import sys

    sys.path.insert(0, ROOT)
    import bench

    assert bench.reduce_max(3.5, torch.device("cpu")) == 3.5
