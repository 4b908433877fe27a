"""Layerwise QK-RMSNorm on rows held in (pinned) host memory, through the
C-ABI's ``qknorm_layerwise_host``.

The library runs the whole pipeline: the batch flows in chunks of tokens
through a ring of device buffers, and the host->device copy of one chunk, the
normalization of the previous one and the device->host copy of the one before
overlap on three streams.  This module only marshals: it keeps, per device,
the two copy streams and a ring for each shape (allocated on first use,
reused by later calls; ``release_buffers()`` frees them), copies gamma to the
device when it is given on the host, and passes pointers and strides.

Calls are asynchronous with respect to the host: they return once the work
is enqueued, and the device's current stream (or ``stream``) reaches the end
of the call when every output row is back in host memory, so
``torch.cuda.current_stream().synchronize()`` (or an event recorded on that
stream) marks completion.  Host tensors must stay alive and unmodified until
then, and should be pinned (``Tensor.pin_memory()``): pageable memory works
but its copies are staged by the driver.  Calls on one device that share a
ring are ordered through that stream; calls must not be issued concurrently
from several host threads.
"""
from __future__ import annotations

import torch

from . import _clib
from ._clib import load as _load

_STREAMS: dict = {}
_RINGS: dict = {}

_DTYPES = {torch.float32: _clib.QKN_F32, torch.bfloat16: _clib.QKN_BF16, torch.float16: _clib.QKN_F16,
           torch.float8_e4m3fn: _clib.QKN_FP8_E4M3}


def release_buffers() -> None:
    """Frees the device rings kept for reuse between calls."""
    _RINGS.clear()


def _copy_streams(device: torch.device):
    key = device.index
    if key not in _STREAMS:
        with torch.cuda.device(key):
            _STREAMS[key] = (torch.cuda.Stream(device=key), torch.cuda.Stream(device=key))
    return _STREAMS[key]


def _ring(device: torch.device, dtype, chunk: int, Hq: int, Hk: int, slots: int) -> torch.Tensor:
    code = _DTYPES[dtype]
    n = _load().qknorm_layerwise_host_ring_bytes(chunk, Hq, Hk, code, slots)
    if n < 0:
        raise ValueError(f"invalid ring shape (chunk_tokens={chunk}, slots={slots})")
    key = (device.index, n)
    ring = _RINGS.get(key)
    if ring is None:
        ring = torch.empty((n,), dtype=torch.uint8, device=device)
        if ring.data_ptr() % 256:
            raise RuntimeError("the device ring must be 256-byte aligned")
        _RINGS[key] = ring
    return ring


def _check_host_rows(t: torch.Tensor, name: str):
    if t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if t.dim() != 2 or (t.shape[0] > 0 and t.shape[1] > 1 and t.stride(1) != 1):
        raise ValueError(f"{name} must be 2-D with unit-stride rows")
    if t.dtype not in _DTYPES:
        raise TypeError(f"{name}: dtype {t.dtype} unsupported")


def _stride(t: torch.Tensor) -> int:
    T, H = t.shape
    return t.stride(0) if T > 1 else max(t.stride(0), H)


def _gamma_on(g: torch.Tensor, device: torch.device, dtype) -> torch.Tensor:
    from . import gamma_dtype
    want = gamma_dtype(dtype)
    if g.dtype != want or g.dim() != 1:
        raise ValueError(f"gamma must be a 1-D {want} tensor")
    return g.to(device, non_blocking=True).contiguous()


def _device(device) -> torch.device:
    d = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    return torch.device("cuda", d.index if d.index is not None else torch.cuda.current_device())


def _call(q_in, q_out, k_in, k_out, q_stride, k_stride, T, Hq, Hk, gamma_q, gamma_k, eps, dtype, device,
          chunk_tokens, slots, stream):
    chunk = min(chunk_tokens, T)
    ring = _ring(device, dtype, chunk, Hq, Hk, slots)
    s_in, s_out = _copy_streams(device)
    main = stream if stream is not None else torch.cuda.current_stream(device)
    with torch.cuda.stream(main):  # gamma reaches the device on the call's stream, ahead of the call
        gq = _gamma_on(gamma_q, device, dtype)
        gk = _gamma_on(gamma_k, device, dtype)
    st = _load().qknorm_layerwise_host(q_in, q_out, gq.data_ptr(), q_stride, k_in, k_out, gk.data_ptr(), k_stride,
                                       T, Hq, Hk, float(eps), _DTYPES[dtype], ring.data_ptr(), ring.numel(), chunk,
                                       main.cuda_stream, s_in.cuda_stream, s_out.cuda_stream)
    _clib.check(st, "qknorm_layerwise_host")


def qknorm_layerwise_host(q_in: torch.Tensor, k_in: torch.Tensor, gamma_q: torch.Tensor,
                          gamma_k: torch.Tensor, eps: float = 1e-6, *, q_out=None, k_out=None,
                          device=None, chunk_tokens: int = 512, slots: int = 3, stream=None):
    """Layerwise QK-Norm of Q rows ``q_in`` [T, Hq] and K rows ``k_in`` [T, Hk]
    held in host memory; results go to host tensors ``q_out`` / ``k_out``
    (allocated pinned and contiguous when None; ``q_out=q_in`` works in place;
    an output has its input's row stride).  gamma may live on the host or
    the device.  Returns ``(q_out, k_out)``."""
    _check_host_rows(q_in, "q_in")
    _check_host_rows(k_in, "k_in")
    T, Hq = q_in.shape
    Tk, Hk = k_in.shape
    if T != Tk or q_in.dtype != k_in.dtype:
        raise ValueError("q_in and k_in must have the same number of tokens and dtype")
    if chunk_tokens < 1 or not 1 <= slots <= 8:
        raise ValueError("chunk_tokens must be >= 1 and slots in [1, 8]")
    device = _device(device)
    if q_out is None:
        q_out = torch.empty_strided((T, Hq), (_stride(q_in), 1), dtype=q_in.dtype, pin_memory=True)
    if k_out is None:
        k_out = torch.empty_strided((T, Hk), (_stride(k_in), 1), dtype=k_in.dtype, pin_memory=True)
    for t, name, src in ((q_out, "q_out", q_in), (k_out, "k_out", k_in)):
        _check_host_rows(t, name)
        if tuple(t.shape) != tuple(src.shape) or t.dtype != src.dtype or (T > 1 and t.stride(0) != src.stride(0)):
            raise ValueError(f"{name} must be a host tensor with the shape, dtype and row stride of its input")
    if T == 0:
        return q_out, k_out
    with torch.cuda.device(device):
        _call(q_in.data_ptr(), q_out.data_ptr(), k_in.data_ptr(), k_out.data_ptr(), _stride(q_in), _stride(k_in),
              T, Hq, Hk, gamma_q, gamma_k, eps, q_in.dtype, device, chunk_tokens, slots, stream)
    return q_out, k_out


def qknorm_packed_host(packed: torch.Tensor, q_col: int, Hq: int, k_col: int, Hk: int,
                       gamma_q: torch.Tensor, gamma_k: torch.Tensor, eps: float = 1e-6, *, out=None,
                       device=None, chunk_tokens: int = 512, slots: int = 3, stream=None):
    """Packed rows (e.g. [Q | K | V]) held in host memory: Q is columns
    [q_col, q_col + Hq) and K columns [k_col, k_col + Hk) of each row of the
    host tensor ``packed`` [T, W] (unit-stride rows).  Only the Q and K
    columns travel; they are normalized on the device and written to the same
    columns of ``out`` (default: ``packed`` itself, in place).  No other
    column of ``packed`` or ``out`` is read or written.  Returns ``out``."""
    _check_host_rows(packed, "packed")
    T, W = packed.shape
    if not (0 <= q_col and q_col + Hq <= W and 0 <= k_col and k_col + Hk <= W) or Hq < 1 or Hk < 1:
        raise ValueError("Q and K columns must lie inside the packed row")
    if chunk_tokens < 1 or not 1 <= slots <= 8:
        raise ValueError("chunk_tokens must be >= 1 and slots in [1, 8]")
    if out is None:
        out = packed
    _check_host_rows(out, "out")
    if tuple(out.shape) != (T, W) or out.dtype != packed.dtype or (T > 1 and out.stride(0) != packed.stride(0)):
        raise ValueError("out must be a host tensor with the shape, dtype and row stride of packed")
    device = _device(device)
    if T == 0:
        return out
    esz = packed.element_size()
    s = _stride(packed)
    with torch.cuda.device(device):
        _call(packed.data_ptr() + q_col * esz, out.data_ptr() + q_col * esz, packed.data_ptr() + k_col * esz,
              out.data_ptr() + k_col * esz, s, s, T, Hq, Hk, gamma_q, gamma_k, eps, packed.dtype, device,
              chunk_tokens, slots, stream)
    return out
