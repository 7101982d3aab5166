"""bench.py's multi-rank plumbing (replicas only): barrier and max-over-ranks timing, checked with
world-size-2 gloo ranks on CPU; and the whole-job rate rule."""
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch
    import bench
    r, w, _ = bench.dist_env()
    d = bench.init_dist(w, "gloo")
    dev = torch.device("cpu")
    bench.barrier(d, dev)
    ms = bench.max_over_ranks(1.5 * (r + 1), d, dev)     # rank-local step times 1.5 and 3.0
    bench.barrier(d, dev)
    d.destroy_process_group()
    q.put((r, ms))


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=10) for _ in range(2))
    assert got == {0: 3.0, 1: 3.0}


def test_whole_job_rate_counts_all_replicas():
    sys.path.insert(0, ROOT)
    import bench
    # 2 replicas of 17.19 GFLOP each, slowest rank 0.06 ms -> 2 * 17.19e9 / 6e-5 FLOP/s
    assert bench.whole_job_rate(17.19e9, 0.06, 2) == pytest.approx(2 * 17.19e9 / 0.06e-3)
    assert bench.whole_job_rate(1.0, 1.0, 1) == pytest.approx(1e3)
