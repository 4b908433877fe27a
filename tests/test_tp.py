"""The tensor-parallel form (the paper's multi-GPU kernel) on one GPU.

``qknorm_tp_layerwise`` runs R ranks, each holding a hidden-dimension shard
of every token's Q and K rows; the ranks exchange only their scalar partial
sums through receive buffers (Phase A) while the shards are multiplied by
gamma (Phase B).  Here all ranks run in one cooperative launch on one GPU,
their receive buffers in that GPU's memory -- the same kernel and protocol a
one-rank-per-GPU deployment uses with peer-mapped buffers.

Every output shard is compared with the oracle's RMS-Norm of the full,
unsharded row (the definition), within the tolerances of the other parity
tests: 1 ulp of the element type, or 1e-5 relative for fp32.  A launch that
leaves one rank out makes the exchange waits run out: the kernel must return,
report the timeout and leave the context usable.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import attention_normalization_b200 as qk
import workloads
from tests.test_parity import ALL_DTYPES, assert_close, oracle_rows

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _batch(T, Hq, Hk, dtype, seed):
    return workloads.random_rows(T, Hq, Hk, dtype, seed=seed, scale=1.5)


def _shards(full: torch.Tensor, R: int):
    w = full.shape[1] // R
    return [full[:, r * w:(r + 1) * w].contiguous().to(DEV) for r in range(R)]


def _gamma_shards(g: torch.Tensor, R: int):
    w = g.numel() // R
    return [g[r * w:(r + 1) * w].contiguous().to(DEV) for r in range(R)]


def run_tp(b, R, ex=None, **kw):
    ex = ex or qk.TpExchange(R, b.T, DEV)
    qo, ko = qk.qknorm_tp_layerwise(_shards(b.q, R), _shards(b.k, R), _gamma_shards(b.gamma_q, R),
                                    _gamma_shards(b.gamma_k, R), b.Hq, b.Hk, b.eps, exchange=ex, **kw)
    torch.cuda.synchronize()
    return torch.cat([q.cpu() for q in qo], dim=1), torch.cat([k.cpu() for k in ko], dim=1)


def check_full(b, q, k):
    yq, eq, _ = oracle_rows(b.q, b.gamma_q, b.eps)
    yk, ek, _ = oracle_rows(b.k, b.gamma_k, b.eps)
    assert_close(q, yq, eq, f"{b.name} TP Q")
    assert_close(k, yk, ek, f"{b.name} TP K")


@pytest.mark.parametrize("dtype", ALL_DTYPES)
@pytest.mark.parametrize("R", [1, 2, 4, 8])
def test_tp_matches_the_full_row_oracle(R, dtype):
    b = _batch(300, 2048, 512, dtype, seed=R)
    q, k = run_tp(b, R)
    check_full(b, q, k)
    assert qk.device_timeouts() == 0


@pytest.mark.parametrize("dtype", ALL_DTYPES)
@pytest.mark.parametrize("R", [2, 4, 8])
def test_tp_system_scope_matches_the_full_row_oracle(R, dtype):
    """The system-scope instantiation -- the one a one-rank-per-GPU deployment
    runs, with system-scope stores and loads on peer memory -- here with every
    rank in one cooperative launch on one GPU, against the oracle."""
    b = _batch(300, 2048, 512, dtype, seed=60 + R)
    q, k = run_tp(b, R, system_scope=True)
    check_full(b, q, k)
    assert qk.device_timeouts() == 0
    gq, gk = run_tp(b, R)  # the GPU-scope instantiation gives the same bits
    assert torch.equal(q, gq) and torch.equal(k, gk)


@pytest.mark.parametrize("R,Hq,Hk,dtype", [
    (2, 8192, 1024, torch.bfloat16),    # 512 + 64 vectors per shard row: the batch-loop form
    (8, 5120, 1024, torch.float32),
])
def test_tp_system_scope_wide_shards(R, Hq, Hk, dtype):
    b = _batch(67, Hq, Hk, dtype, seed=70 + R)
    q, k = run_tp(b, R, system_scope=True)
    check_full(b, q, k)
    assert qk.device_timeouts() == 0


@pytest.mark.parametrize("R,Hq,Hk,dtype", [
    (1, 16384, 2048, torch.bfloat16),   # 2048 + 256 vectors per shard row: 64 per lane, in 16 batches
    (2, 8192, 1024, torch.float32),     # 2048 + 256 vectors per shard row
    (4, 5120, 1024, torch.float8_e4m3fn),
])
def test_tp_wide_shards(R, Hq, Hk, dtype):
    """Shard rows of any width pass through a warp in batches."""
    b = _batch(67, Hq, Hk, dtype, seed=40 + R)
    q, k = run_tp(b, R)
    check_full(b, q, k)
    assert qk.device_timeouts() == 0


def test_tp_prefill_full_size():
    """The prefill batch (T=4096, Hq=Hk=4096 bf16) split over 4 ranks."""
    b = workloads.prefill_bf16()
    q, k = run_tp(b, 4)
    check_full(b, q, k)
    assert qk.device_timeouts() == 0


def test_tp_any_block_count_gives_the_same_bits_and_buffers_are_reused():
    """The result does not depend on how many blocks each rank runs; one
    exchange serves consecutive calls (a new epoch each), in place too."""
    b = _batch(257, 1024, 256, torch.bfloat16, seed=11)
    ex = qk.TpExchange(4, b.T, DEV)
    ref_q, ref_k = run_tp(b, 4, ex)
    for G in (1, 7, 64):
        q, k = run_tp(b, 4, ex, blocks_per_rank=G)
        assert torch.equal(q, ref_q) and torch.equal(k, ref_k)
    qs, ks = _shards(b.q, 4), _shards(b.k, 4)
    qk.qknorm_tp_layerwise(qs, ks, _gamma_shards(b.gamma_q, 4), _gamma_shards(b.gamma_k, 4), b.Hq, b.Hk, b.eps,
                           exchange=ex, in_place=True)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([q.cpu() for q in qs], 1), ref_q)
    assert torch.equal(torch.cat([k.cpu() for k in ks], 1), ref_k)
    check_full(b, ref_q, ref_k)
    assert qk.device_timeouts() == 0


def test_tp_missing_rank_times_out_and_the_context_stays_usable():
    """Ranks 0..2 of a 4-rank group run; rank 3 never publishes, so every
    exchange wait runs out (50 ms): the kernel returns, reports code 4, and
    writes none of the tokens.  A complete call afterwards is correct."""
    R = 4
    b = _batch(64, 1024, 512, torch.bfloat16, seed=12)
    ex = qk.TpExchange(R, b.T, DEV)
    qs, ks = _shards(b.q, R), _shards(b.k, R)
    gq, gk = _gamma_shards(b.gamma_q, R), _gamma_shards(b.gamma_k, R)
    sentinel = [torch.full_like(q, 3.0) for q in qs[:3]]
    qo, _ = qk.qknorm_tp_layerwise(qs[:3], ks[:3], gq[:3], gk[:3], b.Hq, b.Hk, b.eps, exchange=ex, R=R,
                                   first_rank=0, q_out=sentinel, timeout_ns=50_000_000)
    torch.cuda.synchronize()
    assert qk.device_timeouts() == 4
    assert all(torch.all(q == 3.0) for q in qo)
    assert qk.device_timeouts() == 0  # reading cleared it
    q, k = run_tp(b, R, ex)
    check_full(b, q, k)
    assert qk.device_timeouts() == 0


def test_tp_timeout_on_fresh_buffers_is_reported_again():
    """An abort belongs to the receive buffers it happened on and that call's
    epoch.  Ranks 0..2 of 4 time out at epoch 1 (code 4); a fresh exchange,
    whose first call is epoch 1 again, repeats that incomplete call: its waits
    must run out and report code 4 in turn -- not give up at once on the
    earlier abort and report nothing.  A complete call on another fresh
    exchange then matches the oracle, and one on the first exchange's next
    epoch too."""
    R = 4
    b = _batch(64, 1024, 512, torch.bfloat16, seed=13)
    qs, ks = _shards(b.q, R), _shards(b.k, R)
    gq, gk = _gamma_shards(b.gamma_q, R), _gamma_shards(b.gamma_k, R)

    def incomplete(ex):
        sentinel = [torch.full_like(q, 3.0) for q in qs[:3]]
        qo, _ = qk.qknorm_tp_layerwise(qs[:3], ks[:3], gq[:3], gk[:3], b.Hq, b.Hk, b.eps, exchange=ex, R=R,
                                       first_rank=0, q_out=sentinel, timeout_ns=50_000_000)
        torch.cuda.synchronize()
        return qo

    first = qk.TpExchange(R, b.T, DEV)
    qo = incomplete(first)
    assert first.epoch == 1 and qk.device_timeouts() == 4
    assert all(torch.all(q == 3.0) for q in qo)
    second = qk.TpExchange(R, b.T, DEV)
    qo = incomplete(second)
    assert second.epoch == 1
    assert qk.device_timeouts() == 4, "the second exchange's waits gave up without reporting"
    assert all(torch.all(q == 3.0) for q in qo)
    assert qk.device_timeouts() == 0
    q, k = run_tp(b, R, qk.TpExchange(R, b.T, DEV))
    check_full(b, q, k)
    q, k = run_tp(b, R, first)  # epoch 2 on the buffers that saw the abort
    check_full(b, q, k)
    assert qk.device_timeouts() == 0


def test_peer_exchange_single_rank_on_the_gpu():
    """TpPeerExchange's CUDA side on one GPU: a one-rank group allocates,
    zeroes and exports its receive buffer through the runtime's IPC calls, and
    a call through it normalizes like the oracle.  (Groups of several ranks
    need one GPU each.)"""
    import socket

    import torch.distributed as dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        b = _batch(64, 1024, 512, torch.bfloat16, seed=31)
        ex = qk.TpPeerExchange(1, b.T)
        assert len(ex.pointers()) == 1
        q, k = run_tp(b, 1, ex)
        check_full(b, q, k)
        q2, k2 = run_tp(b, 1, ex)  # the next epoch on the same buffer
        assert torch.equal(q, q2) and torch.equal(k, k2)
        assert ex.epoch == 2
        ex.close()
        assert qk.device_timeouts() == 0
    finally:
        dist.destroy_process_group()


def _ipc_pair_worker(rank, port, out):
    import numpy as np
    import torch.distributed as dist
    from cuda.bindings import runtime as rt
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=2)
    try:
        ex = qk.TpPeerExchange(2, 64)
        ptrs = ex.pointers()
        # write a marker into the other rank's buffer through its mapping
        mark = np.array([0x1234 + rank], dtype=np.uint64)
        (err,) = rt.cudaMemcpy(ptrs[1 - rank] + 8 * rank, mark.ctypes.data, 8, rt.cudaMemcpyKind.cudaMemcpyHostToDevice)
        assert err == rt.cudaError_t.cudaSuccess
        (err,) = rt.cudaDeviceSynchronize()
        dist.barrier()
        got = np.zeros(2, dtype=np.uint64)
        (err,) = rt.cudaMemcpy(got.ctypes.data, ptrs[rank], 16, rt.cudaMemcpyKind.cudaMemcpyDeviceToHost)
        assert err == rt.cudaError_t.cudaSuccess
        dist.barrier()  # no rank unmaps while the other may still write
        ex.close()
        out.put((rank, [int(v) for v in got]))
    finally:
        dist.destroy_process_group()


def test_peer_exchange_maps_another_process_buffer():
    """Two processes on this GPU exchange IPC handles through a gloo group and
    each writes a marker into the other's receive buffer through its mapping
    (plain copies; no kernel waits on another process)."""
    import socket

    import torch.multiprocessing as mp
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_ipc_pair_worker, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=180) for _ in range(2))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    # rank r's buffer holds the other rank's marker at that rank's slot, zero elsewhere
    assert got[0] == [0, 0x1234 + 1]
    assert got[1] == [0x1234 + 0, 0]
