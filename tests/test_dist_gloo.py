"""Replica timing across ranks (bench.py's multi-GPU plumbing) on two CPU ranks over gloo."""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    d = bench.Dist(world, backend="gloo")
    my_ms = [10.0, 12.5, 11.0, 9.0][rank]
    d.barrier()
    worst = d.max(my_ms)
    value = bench.throughput(2.0e12, 100, worst, d.world, 1e12)
    out.put((rank, worst, value))
    d.close()


@pytest.mark.parametrize("world", [2, 4])
def test_replica_timing_takes_max_over_ranks(world):
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
    worst = max([10.0, 12.5, 11.0, 9.0][:world])
    for rank, got, value in res:
        assert got == worst
        assert value == pytest.approx(world * 2.0e12 * 100 / (worst * 1e-3) / 1e12)


def test_single_process_needs_no_group():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    env = {k: os.environ.pop(k) for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK") if k in os.environ}
    try:
        d = bench.Dist(1, backend="gloo")
        assert d.max(3.5) == 3.5 and d.pg is None
        with pytest.raises(SystemExit):
            bench.Dist(2, backend="gloo")
    finally:
        os.environ.update(env)
