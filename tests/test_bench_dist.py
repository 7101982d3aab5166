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


def test_bench_helpers_read_peaks_and_profile_traffic():
    """bench.py's host helpers: measured peaks are found, each committed ncu summary gives a
    per-launch traffic figure, and the module defines every name its GPU path uses."""
    import ast
    import builtins
    import bench
    peaks, how = bench.load_peaks()
    assert how in ("measured", "fallback") and peaks["hbm_gbs"] > 0 and peaks["bf16_tflops"] > 0
    assert bench.profile_traffic("prefill_tc_c2") > 0
    assert bench.profile_traffic("decode_split_c4") > 0
    assert bench.profile_traffic("no_such_profile") is None
    tree = ast.parse(open(bench.__file__).read())
    defined = set(dir(builtins)) | {"__file__"}
    for node in ast.walk(tree):
        if isinstance(node, (ast.FunctionDef, ast.ClassDef)):
            defined.add(node.name)
        elif isinstance(node, (ast.Import, ast.ImportFrom)):
            defined.update((a.asname or a.name).split(".")[0] for a in node.names)
        elif isinstance(node, ast.Name) and isinstance(node.ctx, (ast.Store, ast.Del)):
            defined.add(node.id)
        elif isinstance(node, ast.arg):
            defined.add(node.arg)
        elif isinstance(node, ast.ExceptHandler) and node.name:
            defined.add(node.name)
    used = {n.id for n in ast.walk(tree) if isinstance(n, ast.Name) and isinstance(n.ctx, ast.Load)}
    assert not (used - defined), sorted(used - defined)


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` times the oracle on the host and prints one JSON line with the
    contract's keys (the small fp32 workload keeps this to seconds)."""
    import json
    import subprocess
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1", "--warmup", "3",
           "--workload", "c1_fp32_B1_H1_S128_D64"]
    r = subprocess.run(cmd, capture_output=True, text=True, cwd=ROOT, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "TFLOP/s"
    assert line["config"]["workload"] == "c1_fp32_B1_H1_S128_D64"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
