"""The benchmark's multi-rank plumbing on CPU: world size 2 over gloo.

Every rank times its own copy of the workload; the job time is the max over
ranks and the throughput counts the units of all ranks.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import bench
    d = bench.Dist()
    d.init("gloo")
    d.barrier()
    t = 10.0 + rank * 5.0             # rank 1 is the slower one
    mx = d.max(t)
    sm = d.sum(float(rank + 1))
    rate = bench.weak_scaling_rate(131072, d.world, mx)
    out.put((rank, mx, sm, rate))
    d.barrier()
    d.close()


def test_two_rank_max_and_weak_scaling():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, sm, rate in res:
        assert mx == 15.0             # max over ranks
        assert sm == 3.0
        assert rate == pytest.approx(131072 * 2 / 0.015)


def test_single_rank_defaults():
    import bench
    d = bench.Dist()
    assert d.world >= 1 and d.max(3.0) == 3.0 and d.sum(2.0) == 2.0
    assert bench.weak_scaling_rate(10, 1, 1000.0) == pytest.approx(10.0)
