"""Multi-process host logic of the benchmark on CPU (gloo, world size 2).

Ranks normalize independent batches (no data-path collective); the only
cross-rank steps are a barrier and the max over ranks of the timed region, and
rank 0 alone prints.  These run without a GPU.
"""
from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, ms_by_rank, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        r = bench.Ranks(dist)
        r.barrier()
        m = r.max(ms_by_rank[rank])
        agg = bench.whole_job(1_000_000, 10, m, r.world)
        out.put((rank, m, agg["value_gbs"], r.world))
        r.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    ms = [3.0, 5.0]
    procs = [ctx.Process(target=_worker, args=(r, world, port, ms, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for rank, m, value, w in got:
        assert w == 2 and m == 5.0  # every rank sees the slowest rank's time
        # 2 ranks x 10 steps x 1 MB in 5 ms -> 4 GB/s whole job
        assert abs(value - 2 * 1e6 / 0.5e-3 / 1e9) < 1e-9


def test_whole_job_single_process():
    import bench
    agg = bench.whole_job(134_234_112, 2000, 52.8, 1)
    assert abs(agg["ms_per_step"] - 0.0264) < 1e-12
    assert abs(agg["value_gbs"] - 134_234_112 / 26.4e-6 / 1e9) < 1e-6


def test_reference_arm_prints_only_on_rank_zero():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "3", "--warmup", "3"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_line_on_rank_zero():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "3", "--warmup", "3",
                        "--workload", "tiny"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
