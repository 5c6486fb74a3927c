"""The benchmark's multi-rank path on CPU: world size 2 over gloo.  Each rank is
an independent replica; the job's time is the max over ranks and its work the
sum over ranks; a rank that never joins makes the others fail on the store
timeout instead of hanging."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    w, r, lr = bench.dist_env()
    assert (w, r, lr) == (world, rank, rank)
    dist = bench.init_dist(world, "gloo")
    secs = [0.25, 0.5][rank]
    units = [100.0, 300.0][rank]
    t, u = bench.aggregate(dist, secs, units)
    bench.barrier(dist)
    dist.destroy_process_group()
    q.put((rank, t, u))


def test_aggregate_two_ranks_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, t, u in res:
        assert t == 0.5 and u == 400.0


def _lonely(port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK="0", WORLD_SIZE="2",
                      LOCAL_RANK="0")
    import datetime

    import torch.distributed as dist
    try:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=3))
        q.put("joined")
    except Exception as exc:  # the missing rank is detected on the host
        q.put("timeout:" + type(exc).__name__)


def test_missing_rank_times_out_on_host():
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_lonely, args=(port, q))
    p.start()
    p.join(120)
    assert p.exitcode == 0
    assert q.get(timeout=10).startswith("timeout")


def test_bench_single_process_aggregate_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.aggregate(None, 1.5, 10.0) == (1.5, 10.0)
