"""Multi-process (gloo, world size 2) tests of the benchmark's host-side rank logic.

The codec shards without any exchange (each rank encodes and attends over
its own batch), so the only cross-rank steps are the barrier and the
max-over-ranks reduction of the timings; these run here on CPU.
"""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    ws, r, local = bench._dist_init()
    assert (ws, r, local) == (world, rank, rank)
    assert dist.get_backend() == "gloo"
    bench._barrier(ws)
    got = bench._max_over_ranks(10.0 * (rank + 1), ws)
    q.put((rank, got))
    dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=5) for _ in range(2))
    assert res == {0: 20.0, 1: 20.0}


def test_reference_arm_prints_one_json_line():
    env = dict(os.environ, PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["unit"] == "GB/s" and j["value"] > 0
    assert j["cpu_baseline"]["kind"] == "oracle" and j["e2e"]["h2d_bytes_per_step"] == 0
    assert j["warmup"] >= 3


def test_bench_gpus_two_spawns_two_ranks_and_one_line():
    """`bench.py --gpus 2` without a launcher starts two ranks itself (gloo here,
    NCCL on GPUs): each takes its own batch seed, the duration is the max over
    ranks, the whole-job value counts both ranks' units, and rank 0 alone
    prints the one JSON line."""
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    env["PYTHONPATH"] = ROOT
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--dry-run"],
                       capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, r.stdout
    j = json.loads(lines[0])
    assert j["n_gpus"] == 2 and j["scaling"] == "weak"
    assert j["max_ms"] == 20.0                           # rank 1 reports 20 ms, rank 0 10 ms
    units = 8 * 8 * 131072                               # B x Hkv x context of the headline workload
    assert j["value"] == 2 * units / 20.0
    assert len(set(j["config"]["per_rank_seeds"])) == 2  # an independent batch per rank
