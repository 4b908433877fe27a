"""Layerwise QK-RMSNorm on rows held in (pinned) host memory.

The batch is cut into chunks of tokens that flow through a small ring of
device buffers on three CUDA streams: while chunk i is normalized by the
library's kernel, chunk i+1 is copied host->device and chunk i-1
device->host, so the two copy directions (separate copy engines, full-duplex
PCIe/NVLink-C2C) and the kernel overlap.  Every element is normalized on the
GPU by the same C-ABI call as ``qknorm_layerwise``; this module only moves
bytes and orders streams.

All calls are asynchronous with respect to the host: they return once the
work is enqueued, and the current CUDA stream of the device is made to wait
for the last copy back, so ``torch.cuda.current_stream().synchronize()`` (or
an event recorded on that stream) marks completion.  Host tensors must stay
alive and unmodified until then.  Host tensors should be pinned
(``Tensor.pin_memory()``); pageable memory works but the copies then stall.

The device ring (``slots`` chunks) is allocated on first use for a given
shape and kept for later calls; ``release_buffers()`` frees it.  Calls on one
device are serialized through its current stream, so they may share a ring;
calls must not be issued concurrently from several host threads.
"""
from __future__ import annotations

import torch

from . import qknorm_layerwise

_STREAMS: dict = {}
_RINGS: dict = {}


def release_buffers() -> None:
    """Frees the device ring buffers kept for reuse between calls."""
    _RINGS.clear()


def _ring(device: torch.device, dtype, shapes, slots: int):
    """Device buffers for `slots` chunks, allocated once per (device, dtype,
    shapes, slots) and reused by later calls.  Reuse is ordered: a call's copy
    streams first wait for the device's current stream, which itself waited
    for the previous call's last copy back."""
    key = (device.index, dtype, tuple(tuple(s) for s in shapes), slots)
    ring = _RINGS.get(key)
    if ring is None:
        ring = [[torch.empty(shape, dtype=dtype, device=device) for shape in shapes] for _ in range(slots)]
        _RINGS[key] = ring
    return ring


def _streams(device: torch.device):
    key = device.index if device.index is not None else torch.cuda.current_device()
    if key not in _STREAMS:
        with torch.cuda.device(key):
            _STREAMS[key] = tuple(torch.cuda.Stream(device=key) for _ in range(3))
    return _STREAMS[key]


def _check_host_rows(t: torch.Tensor, name: str):
    if t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if t.dim() != 2 or (t.shape[0] > 0 and t.shape[1] > 1 and t.stride(1) != 1):
        raise ValueError(f"{name} must be 2-D with unit-stride rows")


def _pipeline(T: int, chunk_tokens: int, slots: int, device, copy_in, compute, copy_out, ring_shapes, dtype):
    """Runs copy_in(slot_views, t0, t1) / compute(slot_views, stream) /
    copy_out(slot_views, t0, t1) for every chunk over a ring of `slots`
    device buffer sets."""
    h2d, comp, d2h = _streams(device)
    main = torch.cuda.current_stream(device)
    for s in (h2d, comp, d2h):
        s.wait_stream(main)  # e.g. gamma copies queued on the main stream
    ring = _ring(device, dtype, ring_shapes, slots)
    free = [None] * slots
    for i, t0 in enumerate(range(0, T, chunk_tokens)):
        t1 = min(T, t0 + chunk_tokens)
        slot = i % slots
        views = [b[: t1 - t0] for b in ring[slot]]
        with torch.cuda.stream(h2d):
            if free[slot] is not None:
                h2d.wait_event(free[slot])
            copy_in(views, t0, t1)
            loaded = torch.cuda.Event()
            loaded.record(h2d)
        with torch.cuda.stream(comp):
            comp.wait_event(loaded)
            compute(views, comp)
            done = torch.cuda.Event()
            done.record(comp)
        with torch.cuda.stream(d2h):
            d2h.wait_event(done)
            copy_out(views, t0, t1)
            free[slot] = torch.cuda.Event()
            free[slot].record(d2h)
    main.wait_stream(d2h)


def qknorm_layerwise_host(q_in: torch.Tensor, k_in: torch.Tensor, gamma_q: torch.Tensor,
                          gamma_k: torch.Tensor, eps: float = 1e-6, *, q_out=None, k_out=None,
                          device=None, chunk_tokens: int = 512, slots: int = 3):
    """Layerwise QK-Norm of Q rows ``q_in`` [T, Hq] and K rows ``k_in`` [T, Hk]
    held in host memory; results go to host tensors ``q_out`` / ``k_out``
    (allocated pinned and contiguous when None; ``q_out=q_in`` works in place).
    gamma may live on the host or the device.  Returns ``(q_out, k_out)``."""
    _check_host_rows(q_in, "q_in")
    _check_host_rows(k_in, "k_in")
    T, Hq = q_in.shape
    Tk, Hk = k_in.shape
    if T != Tk or q_in.dtype != k_in.dtype:
        raise ValueError("q_in and k_in must have the same number of tokens and dtype")
    if chunk_tokens < 1 or slots < 2:
        raise ValueError("chunk_tokens must be >= 1 and slots >= 2")
    device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    if q_out is None:
        q_out = torch.empty((T, Hq), dtype=q_in.dtype, pin_memory=True)
    if k_out is None:
        k_out = torch.empty((T, Hk), dtype=k_in.dtype, pin_memory=True)
    for t, name, shape in ((q_out, "q_out", (T, Hq)), (k_out, "k_out", (T, Hk))):
        _check_host_rows(t, name)
        if tuple(t.shape) != shape or t.dtype != q_in.dtype:
            raise ValueError(f"{name} must be a host tensor of shape {shape} and dtype {q_in.dtype}")
    if T == 0:
        return q_out, k_out
    with torch.cuda.device(device):
        gq = gamma_q.to(device, non_blocking=True)
        gk = gamma_k.to(device, non_blocking=True)
        chunk = min(chunk_tokens, T)

        def copy_in(v, t0, t1):
            v[0].copy_(q_in[t0:t1], non_blocking=True)
            v[1].copy_(k_in[t0:t1], non_blocking=True)

        def compute(v, stream):
            qknorm_layerwise(v[0], v[1], gq, gk, eps, q_out=v[0], k_out=v[1], stream=stream)

        def copy_out(v, t0, t1):
            q_out[t0:t1].copy_(v[0], non_blocking=True)
            k_out[t0:t1].copy_(v[1], non_blocking=True)

        _pipeline(T, chunk, slots, device, copy_in, compute, copy_out, [(chunk, Hq), (chunk, Hk)], q_in.dtype)
        comp = _streams(device)[1]
        gq.record_stream(comp)
        gk.record_stream(comp)
    return q_out, k_out


def qknorm_packed_host(packed: torch.Tensor, q_col: int, Hq: int, k_col: int, Hk: int,
                       gamma_q: torch.Tensor, gamma_k: torch.Tensor, eps: float = 1e-6, *, out=None,
                       device=None, chunk_tokens: int = 512, slots: int = 3):
    """Packed rows (e.g. [Q | K | V]) held in host memory: Q is columns
    [q_col, q_col + Hq) and K columns [k_col, k_col + Hk) of each row of the
    contiguous host tensor ``packed`` [T, W].  Whole rows travel; Q and K are
    normalized in place on the device and the rows come back into ``out``
    (default: ``packed`` itself), every other column unchanged."""
    _check_host_rows(packed, "packed")
    if not packed.is_contiguous():
        raise ValueError("packed must be contiguous")
    T, W = packed.shape
    if not (0 <= q_col and q_col + Hq <= W and 0 <= k_col and k_col + Hk <= W):
        raise ValueError("Q and K columns must lie inside the packed row")
    if chunk_tokens < 1 or slots < 2:
        raise ValueError("chunk_tokens must be >= 1 and slots >= 2")
    if out is None:
        out = packed
    if tuple(out.shape) != (T, W) or out.dtype != packed.dtype or out.is_cuda or not out.is_contiguous():
        raise ValueError("out must be a contiguous host tensor like packed")
    device = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    if T == 0:
        return out
    with torch.cuda.device(device):
        gq = gamma_q.to(device, non_blocking=True)
        gk = gamma_k.to(device, non_blocking=True)
        chunk = min(chunk_tokens, T)

        def copy_in(v, t0, t1):
            v[0].copy_(packed[t0:t1], non_blocking=True)

        def compute(v, stream):
            rows = v[0]
            q = rows[:, q_col:q_col + Hq]
            k = rows[:, k_col:k_col + Hk]
            qknorm_layerwise(q, k, gq, gk, eps, q_out=q, k_out=k, stream=stream)

        def copy_out(v, t0, t1):
            out[t0:t1].copy_(v[0], non_blocking=True)

        _pipeline(T, chunk, slots, device, copy_in, compute, copy_out, [(chunk, W)], packed.dtype)
        comp = _streams(device)[1]
        gq.record_stream(comp)
        gk.record_stream(comp)
    return out
