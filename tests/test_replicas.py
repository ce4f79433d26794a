"""The multi-GPU path of bench.py is independent replicas (sequences and their
caches never cross GPUs, so there is no data-path collective). Its host-side
plumbing -- rank discovery, the barrier around the timed region, the max of
the timed region over ranks and the whole-job throughput -- is exercised here
with world_size 2 over gloo on the CPU."""
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q):
    sys.path.insert(0, ROOT)
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import datetime
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w, r, local = bench.dist_env()
        bench.barrier(w)
        t_ms = 10.0 * (r + 1)                 # rank 1 is the slow one
        t_max = bench.max_over_ranks(t_ms, w)
        value = bench.replica_throughput(1000, t_max, w)
        bench.barrier(w)
        q.put((r, w, local, t_max, value))
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank_and_sum_the_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(2))
    for r, (rank, world, local, t_max, value) in enumerate(got):
        assert (rank, world, local) == (r, 2, r)
        assert t_max == 20.0
        # 2 replicas x 1000 units in 20 ms
        assert value == pytest.approx(2 * 1000 / 0.020)


def test_single_process_defaults():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.replica_throughput(10, 1000.0, 1) == pytest.approx(10.0)
