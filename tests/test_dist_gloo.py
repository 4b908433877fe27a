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


# --------------------------------------------------------------------------- one rank per GPU: receive buffers

class FakeIpc:
    """Stands in for CUDA IPC on CPU: a rank's buffer is a made-up address, a
    handle names the exporting address, and opening maps it to an address of
    its own; every call is recorded."""

    def __init__(self, rank):
        self.rank = rank
        self.log = []

    def alloc_zeroed(self, nbytes):
        self.log.append(("alloc", nbytes))
        return 0x10000000 * (self.rank + 1)

    def free(self, ptr):
        self.log.append(("free", ptr))

    def export(self, ptr):
        self.log.append(("export", ptr))
        return ptr.to_bytes(8, "little") + bytes(56)

    def open(self, handle):
        ptr = int.from_bytes(handle[:8], "little")
        self.log.append(("open", ptr))
        return ptr + 0x700000000000

    def close(self, ptr):
        self.log.append(("close", ptr))


def _peer_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from attention_normalization_b200.tp_peer import TpPeerExchange
        ipc = FakeIpc(rank)
        ex = TpPeerExchange(world, 4096, ipc=ipc)
        ptrs = ex.pointers()
        epochs = [ex.next_epoch(), ex.next_epoch()]
        ex.close()
        out.put((rank, ptrs, epochs, ipc.log))
    finally:
        dist.destroy_process_group()


def test_peer_exchange_handles_gloo():
    """Each rank allocates and exports its buffer, opens every other rank's
    handle in rank order, keeps its own at its rank; epochs step from 1 on
    every rank; close unmaps the peers and frees its own buffer."""
    world, port = 3, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_peer_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    own = [0x10000000 * (r + 1) for r in range(world)]
    for rank, ptrs, epochs, log in got:
        assert epochs == [1, 2]
        assert ptrs == [own[r] if r == rank else own[r] + 0x700000000000 for r in range(world)]
        assert log[0] == ("alloc", world * 4096 * 16 + 16) and log[1] == ("export", own[rank])  # + abort-word trailer
        assert [e for e in log if e[0] == "open"] == [("open", own[r]) for r in range(world) if r != rank]
        assert [e for e in log if e[0] == "close"] == [("close", own[r] + 0x700000000000)
                                                      for r in range(world) if r != rank]
        assert log[-1] == ("free", own[rank])


def _peer_bad_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from attention_normalization_b200.tp_peer import TpPeerExchange
        try:
            TpPeerExchange(world + 1, 16, ipc=FakeIpc(rank))
            out.put((rank, "accepted"))
        except ValueError as e:
            out.put((rank, str(e)))
    finally:
        dist.destroy_process_group()


def test_peer_exchange_rejects_a_group_of_another_size_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_peer_bad_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert all("R = 3" in msg for _, msg in got)
