"""Layerwise QK-RMSNorm for NVIDIA B200 (sm_100a).

Python binding over the C-ABI library ``libqknorm.so`` (include/qknorm.h).  The
functions here only marshal torch CUDA tensors into pointers, strides and a
stream; every step of the computation runs in the library's CUDA kernels.  If
the library is missing the call raises — there is no CPU path.

RMS-Norm over the full projected Q and K rows of each token ("SwiftQK: Fast and
Communication-Efficient Tensor Parallelism for Query-Key Normalization",
Background, Equation 1):  y = x / sqrt(mean(x^2) + eps) * gamma, and its Phase A
shard decomposition (per-shard squared sums, fp32 aggregation, then scaling).

Tensors: 2-D ``[T, width]`` views whose rows may be strided (``stride(1) == 1``,
``stride(0) >= width``), e.g. Q and K views into a packed ``[T, Hq+Hk+Hv]``
buffer.  An output has the same row stride as its input (the C-ABI takes one
stride per tensor); pass ``q_out=q_in`` to normalize in place.
"""
from __future__ import annotations

import ctypes

import torch

from . import _clib
from ._clib import QknLaunch, QKNormError

__all__ = ["qknorm_layerwise", "qknorm_headwise", "qknorm_qkv_gemm_stats", "qknorm_qkv_projection",
           "qkv_workspace_bytes", "device_timeouts", "qknorm_tp_layerwise", "TpExchange", "TpPeerExchange",
           "qknorm_partial_stats", "qknorm_combine_apply", "qknorm_partial_stats_shards",
           "qknorm_combine_apply_shards", "gamma_dtype",
           "qknorm_layerwise_plan", "qknorm_layerwise_host", "qknorm_packed_host",
           "plan_shape", "plan_grid", "regions_overlap", "qkv_gemm_schedule", "qkv_gemm_plan", "capi", "version", "QknLaunch", "QKNormError"]

_DTYPES = {torch.float32: _clib.QKN_F32, torch.bfloat16: _clib.QKN_BF16, torch.float16: _clib.QKN_F16,
           torch.float8_e4m3fn: _clib.QKN_FP8_E4M3}


def gamma_dtype(dtype: torch.dtype) -> torch.dtype:
    """The gamma type that goes with activations of `dtype` (bf16 for E4M3)."""
    return torch.bfloat16 if dtype == torch.float8_e4m3fn else dtype


def capi() -> ctypes.CDLL:
    """The raw C-ABI (functions take pointers and sizes, as in include/qknorm.h)."""
    return _clib.load()


def version() -> int:
    return capi().qknorm_version()



# --------------------------------------------------------------------------- marshalling

def _rows(t: torch.Tensor, name: str):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (this library has no CPU path)")
    if t.dtype not in _DTYPES:
        raise TypeError(f"{name}: dtype {t.dtype} unsupported (float32, bfloat16, float16, float8_e4m3fn)")
    shape = t.shape
    if len(shape) != 2:
        raise ValueError(f"{name} must be 2-D [T, width]")
    T, H = shape
    s0, s1 = t.stride()
    if T > 0 and H > 1 and s1 != 1:
        raise ValueError(f"{name} rows must be unit-stride along the width")
    return T, H, (s0 if T > 1 else max(s0, H))


def _vec(t: torch.Tensor, name: str, n: int, dtype: torch.dtype, device):
    if not (isinstance(t, torch.Tensor) and t.is_cuda and t.dtype == dtype and t.is_contiguous()
            and t.numel() == n and t.device == device):
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor of {n} elements on {device}")
    return t.data_ptr()


def _out_like(x: torch.Tensor, stride: int) -> torch.Tensor:
    T, H = x.shape
    return torch.empty_strided((T, H), (stride, 1), dtype=x.dtype, device=x.device)


# The current stream's raw handle without building a Stream object (a
# fraction of a microsecond instead of about two per call), where torch has it.
_raw_current_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream_handle(stream, device) -> int:
    if stream is None:
        if _raw_current_stream is not None:
            return _raw_current_stream(device.index if device.index is not None else torch.cuda.current_device())
        return torch.cuda.current_stream(device).cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


class _NoSwitch:
    def __enter__(self):
        return None

    def __exit__(self, *exc):
        return False


_NO_SWITCH = _NoSwitch()


def _on(device):
    """Makes `device` current for a call: a no-op when it already is (the
    usual case), else torch.cuda.device."""
    if device.index is None or device.index == torch.cuda.current_device():
        return _NO_SWITCH
    return torch.cuda.device(device)


def _same(dev_a, dtype_a, t: torch.Tensor, name: str):
    if t.device != dev_a or t.dtype != dtype_a:
        raise ValueError(f"{name} must be on {dev_a} with dtype {dtype_a}")


def _layerwise_args(q_in, k_in, gamma_q, gamma_k, eps, q_out, k_out):
    Tq, Hq, sq = _rows(q_in, "q_in")
    Tk, Hk, sk = _rows(k_in, "k_in")
    if Tq != Tk:
        raise ValueError(f"q_in and k_in must have the same number of tokens ({Tq} != {Tk})")
    dev, dt = q_in.device, q_in.dtype
    _same(dev, dt, k_in, "k_in")
    if q_out is None:
        q_out = _out_like(q_in, sq)
    if k_out is None:
        k_out = _out_like(k_in, sk)
    for t, name, (T, H, s) in ((q_out, "q_out", (Tq, Hq, sq)), (k_out, "k_out", (Tk, Hk, sk))):
        _same(dev, dt, t, name)
        To, Ho, so = _rows(t, name)
        if (To, Ho) != (T, H) or (T > 1 and so != s):
            raise ValueError(f"{name} must match its input's shape and row stride")
    gdt = gamma_dtype(dt)
    args = [q_in.data_ptr(), q_out.data_ptr(), _vec(gamma_q, "gamma_q", Hq, gdt, dev), sq,
            k_in.data_ptr(), k_out.data_ptr(), _vec(gamma_k, "gamma_k", Hk, gdt, dev), sk,
            Tq, Hq, Hk, float(eps), _DTYPES[dt]]
    return args, q_out, k_out, dev


# --------------------------------------------------------------------------- API

def qknorm_layerwise(q_in: torch.Tensor, k_in: torch.Tensor, gamma_q: torch.Tensor,
                     gamma_k: torch.Tensor, eps: float = 1e-6, *, q_out=None, k_out=None,
                     stream=None, launch: QknLaunch | dict | None = None):
    """Fused layerwise QK-Norm of all tokens in one launch; returns ``(q_out, k_out)``.

    ``launch`` pins a launch shape (``qkn_launch``); every valid shape agrees
    with the default within one unit in the last place (the squared sum is
    added in a shape-dependent order) and is deterministic run to run.
    Asynchronous on ``stream`` (default: the current stream).
    """
    args, q_out, k_out, dev = _layerwise_args(q_in, k_in, gamma_q, gamma_k, eps, q_out, k_out)
    lib = capi()
    with _on(dev):
        s = _stream_handle(stream, dev)
        if launch is None:
            st = lib.qknorm_layerwise(*args, s)
        else:
            st = lib.qknorm_layerwise_launch(*args, s, ctypes.byref(_launch_struct(launch)))
    _clib.check(st, "qknorm_layerwise")
    return q_out, k_out


def qknorm_headwise(q_in: torch.Tensor, k_in: torch.Tensor, gamma_q: torch.Tensor, gamma_k: torch.Tensor,
                    head_dim: int, eps: float = 1e-6, *, q_out=None, k_out=None, stream=None,
                    launch: QknLaunch | dict | None = None):
    """Headwise QK-Norm: every head of ``head_dim`` elements in the Q rows
    ``[T, q_heads * head_dim]`` and K rows ``[T, k_heads * head_dim]`` is
    normalized on its own, gamma ``[head_dim]`` shared by a tensor's heads.
    One launch for Q and K; returns ``(q_out, k_out)``."""
    Tq, Wq, sq = _rows(q_in, "q_in")
    Tk, Wk, sk = _rows(k_in, "k_in")
    if Tq != Tk:
        raise ValueError("q_in and k_in must have the same number of tokens")
    if head_dim < 1 or Wq % head_dim or Wk % head_dim:
        raise ValueError("row widths must be whole numbers of heads of head_dim elements")
    dev, dt = q_in.device, q_in.dtype
    _same(dev, dt, k_in, "k_in")
    if q_out is None:
        q_out = _out_like(q_in, sq)
    if k_out is None:
        k_out = _out_like(k_in, sk)
    for t, name, (T, W, s) in ((q_out, "q_out", (Tq, Wq, sq)), (k_out, "k_out", (Tk, Wk, sk))):
        _same(dev, dt, t, name)
        To, Wo, so = _rows(t, name)
        if (To, Wo) != (T, W) or (T > 1 and so != s):
            raise ValueError(f"{name} must match its input's shape and row stride")
    gdt = gamma_dtype(dt)
    args = [q_in.data_ptr(), q_out.data_ptr(), _vec(gamma_q, "gamma_q", head_dim, gdt, dev), sq, Wq // head_dim,
            k_in.data_ptr(), k_out.data_ptr(), _vec(gamma_k, "gamma_k", head_dim, gdt, dev), sk, Wk // head_dim,
            Tq, int(head_dim), float(eps), _DTYPES[dt]]
    with _on(dev):
        s = _stream_handle(stream, dev)
        if launch is None:
            st = capi().qknorm_headwise(*args, s)
        else:
            st = capi().qknorm_headwise_launch(*args, s, ctypes.byref(_launch_struct(launch)))
    _clib.check(st, "qknorm_headwise")
    return q_out, k_out


# --------------------------------------------------------------------------- QKV projection

QKV_TILE_N = 256  # output columns per GEMM tile = per partial sum


def _projection_args(x, w, Hq, Hk, Hv, qkv):
    T, D, xs = _rows(x, "x")
    N, Dw, ws = _rows(w, "w")
    if x.dtype != torch.bfloat16 or w.dtype != torch.bfloat16:
        raise TypeError("the projection takes bfloat16 x and w")
    if Dw != D:
        raise ValueError(f"w must be [Hq + Hk + Hv, D] with D = {D}, got width {Dw}")
    if N != Hq + Hk + Hv:
        raise ValueError(f"w has {N} rows, Hq + Hk + Hv = {Hq + Hk + Hv}")
    _same(x.device, x.dtype, w, "w")
    if qkv is None:
        qkv = torch.empty((T, N), dtype=x.dtype, device=x.device)
    _same(x.device, x.dtype, qkv, "qkv")
    To, No, qs = _rows(qkv, "qkv")
    if (To, No) != (T, N):
        raise ValueError(f"qkv must be [{T}, {N}]")
    return T, D, xs, ws, qkv, qs


def qkv_workspace_bytes(T: int, Hq: int, Hk: int) -> int:
    """Workspace ``qknorm_qkv_projection`` needs (the per-tile partial sums)."""
    n = capi().qknorm_qkv_projection_workspace_bytes(T, Hq, Hk)
    if n < 0:
        raise ValueError("invalid sizes for the projection workspace")
    return n


def qknorm_qkv_gemm_stats(x: torch.Tensor, w: torch.Tensor, Hq: int, Hk: int, Hv: int, *, qkv=None,
                          q_sums=None, k_sums=None, stream=None):
    """QKV projection ``qkv = bf16(x @ w.T)`` on the tensor cores, with the
    squared sum of every 256-column Q and K tile of each token written by the
    epilogue.  Returns ``(qkv, q_sums [Hq/256, T], k_sums [Hk/256, T])``."""
    T, D, xs, ws, qkv, qs = _projection_args(x, w, Hq, Hk, Hv, qkv)
    dev = x.device
    if q_sums is None:
        q_sums = torch.empty((Hq // QKV_TILE_N, T), dtype=torch.float32, device=dev)
    if k_sums is None:
        k_sums = torch.empty((Hk // QKV_TILE_N, T), dtype=torch.float32, device=dev)
    for t, name, rows in ((q_sums, "q_sums", Hq // QKV_TILE_N), (k_sums, "k_sums", Hk // QKV_TILE_N)):
        if not (t.is_cuda and t.device == dev and t.dtype == torch.float32 and t.is_contiguous()
                and t.numel() == rows * T):
            raise ValueError(f"{name} must be a contiguous float32 CUDA tensor of {rows} x {T}")
    with _on(dev):
        st = capi().qknorm_qkv_gemm_stats(x.data_ptr(), xs, w.data_ptr(), ws, qkv.data_ptr(), qs, T, D, Hq, Hk, Hv,
                                          q_sums.data_ptr(), k_sums.data_ptr(), _clib.QKN_BF16,
                                          _stream_handle(stream, dev))
    _clib.check(st, "qknorm_qkv_gemm_stats")
    return qkv, q_sums, k_sums


def qknorm_qkv_projection(x: torch.Tensor, w: torch.Tensor, gamma_q: torch.Tensor, gamma_k: torch.Tensor,
                          Hq: int, Hk: int, Hv: int, eps: float = 1e-6, *, qkv=None, workspace=None, stream=None):
    """QKV projection followed by layerwise QK-Norm of its Q and K columns
    (partial sums from the GEMM epilogue, then combine and scale in place).
    Returns ``qkv [T, Hq + Hk + Hv]``."""
    T, D, xs, ws, qkv, qs = _projection_args(x, w, Hq, Hk, Hv, qkv)
    dev = x.device
    need = qkv_workspace_bytes(T, Hq, Hk) if Hq % QKV_TILE_N == 0 and Hk % QKV_TILE_N == 0 else 0
    if workspace is None:
        workspace = torch.empty((max(need, 4) // 4,), dtype=torch.float32, device=dev)
    if not (workspace.is_cuda and workspace.device == dev and workspace.is_contiguous()):
        raise ValueError("workspace must be a contiguous CUDA tensor on the device of x")
    gq = _vec(gamma_q, "gamma_q", Hq, torch.bfloat16, dev)
    gk = _vec(gamma_k, "gamma_k", Hk, torch.bfloat16, dev)
    with _on(dev):
        st = capi().qknorm_qkv_projection(x.data_ptr(), xs, w.data_ptr(), ws, qkv.data_ptr(), qs, gq, gk, T, D,
                                          Hq, Hk, Hv, float(eps), workspace.data_ptr(),
                                          workspace.numel() * workspace.element_size(), _clib.QKN_BF16,
                                          _stream_handle(stream, dev))
    _clib.check(st, "qknorm_qkv_projection")
    return qkv


def device_timeouts(device=None) -> int:
    """Synchronize ``device`` and return (and clear) the code a bounded wait in
    the projection kernel recorded: 0 when none ran out."""
    code = ctypes.c_int32(0)
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        _clib.check(capi().qknorm_device_timeouts(ctypes.byref(code)), "qknorm_device_timeouts")
    return code.value


# --------------------------------------------------------------------------- tensor-parallel form

class TpExchange:
    """Receive buffers of an R-rank tensor-parallel group, all on one device
    (the single-GPU form, where one call runs every rank), and the call epoch.
    Each buffer holds [R][T][2] 64-bit words; they start zeroed and every call
    takes the next epoch, so they are never cleared again."""

    def __init__(self, R: int, T: int, device):
        n = capi().qknorm_tp_recv_bytes(R, T)
        if n < 0:
            raise ValueError(f"invalid R={R} or T={T} for the exchange")
        self.R, self.T = R, T
        self.buffers = [torch.zeros((max(n, 8) // 8,), dtype=torch.int64, device=device) for _ in range(R)]
        self.epoch = 0

    def pointers(self):
        return [b.data_ptr() for b in self.buffers]

    def next_epoch(self) -> int:
        self.epoch += 1
        if self.epoch >= 2 ** 32:
            raise RuntimeError("exchange epochs exhausted; make a new TpExchange")
        return self.epoch


from .tp_peer import TpPeerExchange  # noqa: E402  (one rank per GPU: receive buffers over CUDA IPC)


def qknorm_tp_layerwise(q_shards, k_shards, gamma_q_shards, gamma_k_shards, Hq_full: int, Hk_full: int,
                        eps: float = 1e-6, *, exchange: TpExchange | TpPeerExchange | None = None, recv=None,
                        epoch: int | None = None,
                        R: int | None = None, first_rank: int = 0, q_out=None, k_out=None, in_place: bool = False,
                        blocks_per_rank: int = 0, timeout_ns: int = 0, system_scope: bool = False, stream=None):
    """Tensor-parallel layerwise QK-Norm: runs ranks first_rank ..
    first_rank + len(q_shards) - 1 of an R-rank group; shard j holds Q columns
    of rank first_rank + j for all T tokens.  The ranks exchange only their
    scalar partial sums (through ``exchange`` / ``recv``): a ``TpExchange``
    when every rank runs in this call on this GPU, a ``TpPeerExchange`` when
    each process runs its own rank on its own GPU (pass ``first_rank`` = that
    rank and one shard).  ``system_scope`` runs the exchange with system-scope
    loads and stores (the peer-memory form) even when every rank is in this
    call.  Returns the lists ``(q_out, k_out)``."""
    n_local = len(q_shards)
    if not (n_local == len(k_shards) == len(gamma_q_shards) == len(gamma_k_shards)) or n_local < 1:
        raise ValueError("one Q shard, K shard and gamma slice each per local rank")
    T, hq, sq = _rows(q_shards[0], "q_shards[0]")
    _, hk, sk = _rows(k_shards[0], "k_shards[0]")
    dev, dt = q_shards[0].device, q_shards[0].dtype
    for j in range(n_local):
        for t, name, (H, s) in ((q_shards[j], f"q_shards[{j}]", (hq, sq)), (k_shards[j], f"k_shards[{j}]", (hk, sk))):
            _same(dev, dt, t, name)
            Tj, Hj, sj = _rows(t, name)
            if (Tj, Hj) != (T, H) or (T > 1 and sj != s):
                raise ValueError(f"{name}: every local shard must have the same shape and row stride")
    if exchange is not None:
        recv = exchange.pointers()
        R = exchange.R if R is None else R
        epoch = exchange.next_epoch() if epoch is None else epoch
    if recv is None or epoch is None:
        raise ValueError("pass an exchange, or recv pointers and an epoch")
    R = n_local if R is None else R
    if len(recv) != R:
        raise ValueError(f"{len(recv)} receive buffers for R={R}")
    if in_place:
        q_out, k_out = list(q_shards), list(k_shards)
    if q_out is None:
        q_out = [_out_like(q, sq) for q in q_shards]
    if k_out is None:
        k_out = [_out_like(k, sk) for k in k_shards]
    gdt = gamma_dtype(dt)
    gq = [_vec(g, f"gamma_q_shards[{j}]", hq, gdt, dev) for j, g in enumerate(gamma_q_shards)]
    gk = [_vec(g, f"gamma_k_shards[{j}]", hk, gdt, dev) for j, g in enumerate(gamma_k_shards)]
    P = ctypes.c_void_p

    def arr(xs):
        return (P * len(xs))(*[int(x) for x in xs])
    with _on(dev):
        st = capi().qknorm_tp_layerwise_scope(R, first_rank, n_local, arr([q.data_ptr() for q in q_shards]),
                                              arr([q.data_ptr() for q in q_out]), arr(gq), sq, hq, int(Hq_full),
                                              arr([k.data_ptr() for k in k_shards]),
                                              arr([k.data_ptr() for k in k_out]), arr(gk), sk, hk, int(Hk_full), T,
                                              float(eps), _DTYPES[dt], arr(recv), int(epoch), int(blocks_per_rank),
                                              int(timeout_ns), 1 if system_scope else 0, _stream_handle(stream, dev))
    _clib.check(st, "qknorm_tp_layerwise")
    return q_out, k_out


def qknorm_layerwise_plan(q_in, k_in, gamma_q, gamma_k, eps: float = 1e-6, *, q_out=None,
                          k_out=None) -> dict:
    """The launch ``qknorm_layerwise`` would use for these tensors."""
    args, _, _, dev = _layerwise_args(q_in, k_in, gamma_q, gamma_k, eps, q_out, k_out)
    L = QknLaunch()
    with _on(dev):
        st = capi().qknorm_layerwise_plan(*args, ctypes.byref(L))
    _clib.check(st, "qknorm_layerwise_plan")
    return L.as_dict()


def qkv_gemm_schedule(T: int, D: int, Hq: int, Hk: int, Hv: int, clusters: int, l2_bytes: int) -> dict:
    """The projection GEMM's schedule for ``clusters`` resident CTA pairs and
    an L2 of ``l2_bytes`` (pure; no GPU needed)."""
    S = _clib.QknGemmSchedule()
    st = capi().qknorm_qkv_gemm_schedule(int(T), int(D), int(Hq), int(Hk), int(Hv), int(clusters), int(l2_bytes),
                                         ctypes.byref(S))
    _clib.check(st, "qknorm_qkv_gemm_schedule")
    return S.as_dict()


def qkv_gemm_plan(T: int, D: int, Hq: int, Hk: int, Hv: int, device=None) -> dict:
    """The schedule the projection entry points use for this shape on
    ``device`` (default: the current CUDA device)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    S = _clib.QknGemmSchedule()
    with _on(dev):
        st = capi().qknorm_qkv_gemm_plan(int(T), int(D), int(Hq), int(Hk), int(Hv), ctypes.byref(S))
    _clib.check(st, "qknorm_qkv_gemm_plan")
    return S.as_dict()


def _launch_struct(launch):
    return launch if isinstance(launch, QknLaunch) else QknLaunch(**launch)


def qknorm_partial_stats(q_shard: torch.Tensor, k_shard: torch.Tensor, q_sumsq=None, k_sumsq=None,
                         *, stream=None, launch: QknLaunch | dict | None = None):
    """Phase A local step: fp32 squared sum of every token's Q-shard and K-shard
    row; returns ``(q_sumsq, k_sumsq)``, each ``[T]`` float32 (a row of a
    caller-owned ``[P, T]`` array may be passed)."""
    T, hq, sq = _rows(q_shard, "q_shard")
    Tk, hk, sk = _rows(k_shard, "k_shard")
    if T != Tk:
        raise ValueError("q_shard and k_shard must have the same number of tokens")
    dev, dt = q_shard.device, q_shard.dtype
    _same(dev, dt, k_shard, "k_shard")
    if q_sumsq is None:
        q_sumsq = torch.empty((T,), dtype=torch.float32, device=dev)
    if k_sumsq is None:
        k_sumsq = torch.empty((T,), dtype=torch.float32, device=dev)
    pq = _vec(q_sumsq, "q_sumsq", T, torch.float32, dev)
    pk = _vec(k_sumsq, "k_sumsq", T, torch.float32, dev)
    args = [q_shard.data_ptr(), sq, hq, pq, k_shard.data_ptr(), sk, hk, pk, T, _DTYPES[dt]]
    with _on(dev):
        s = _stream_handle(stream, dev)
        if launch is None:
            st = capi().qknorm_partial_stats(*args, s)
        else:
            st = capi().qknorm_partial_stats_launch(*args, s, ctypes.byref(_launch_struct(launch)))
    _clib.check(st, "qknorm_partial_stats")
    return q_sumsq, k_sumsq


def qknorm_combine_apply(q_in: torch.Tensor, k_in: torch.Tensor, gamma_q_shard: torch.Tensor,
                         gamma_k_shard: torch.Tensor, q_sumsq_all: torch.Tensor,
                         k_sumsq_all: torch.Tensor, Hq_full: int, Hk_full: int, eps: float = 1e-6,
                         *, q_out=None, k_out=None, stream=None, launch: QknLaunch | dict | None = None):
    """Phase A aggregation of the ``[P, T]`` fp32 partial sums (order p = 0..P-1),
    factor over the FULL widths, then scale this shard; returns ``(q_out, k_out)``."""
    T, hq, sq = _rows(q_in, "q_in")
    Tk, hk, sk = _rows(k_in, "k_in")
    if T != Tk:
        raise ValueError("q_in and k_in must have the same number of tokens")
    dev, dt = q_in.device, q_in.dtype
    _same(dev, dt, k_in, "k_in")
    if q_sumsq_all.dim() != 2 or k_sumsq_all.dim() != 2 or q_sumsq_all.shape != k_sumsq_all.shape \
            or q_sumsq_all.shape[1] != T:
        raise ValueError("q_sumsq_all and k_sumsq_all must both be [P, T]")
    P = q_sumsq_all.shape[0]
    ps_q = _vec(q_sumsq_all, "q_sumsq_all", P * T, torch.float32, dev)
    ps_k = _vec(k_sumsq_all, "k_sumsq_all", P * T, torch.float32, dev)
    if q_out is None:
        q_out = _out_like(q_in, sq)
    if k_out is None:
        k_out = _out_like(k_in, sk)
    for t, name, (H, s) in ((q_out, "q_out", (hq, sq)), (k_out, "k_out", (hk, sk))):
        _same(dev, dt, t, name)
        To, Ho, so = _rows(t, name)
        if (To, Ho) != (T, H) or (T > 1 and so != s):
            raise ValueError(f"{name} must match its input's shape and row stride")
    gdt = gamma_dtype(dt)
    args = [q_in.data_ptr(), q_out.data_ptr(), _vec(gamma_q_shard, "gamma_q_shard", hq, gdt, dev), sq, hq,
            ps_q, int(Hq_full),
            k_in.data_ptr(), k_out.data_ptr(), _vec(gamma_k_shard, "gamma_k_shard", hk, gdt, dev), sk, hk,
            ps_k, int(Hk_full), P, T, float(eps), _DTYPES[dt]]
    with _on(dev):
        s = _stream_handle(stream, dev)
        if launch is None:
            st = capi().qknorm_combine_apply(*args, s)
        else:
            st = capi().qknorm_combine_apply_launch(*args, s, ctypes.byref(_launch_struct(launch)))
    _clib.check(st, "qknorm_combine_apply")
    return q_out, k_out


def _ptr_array(xs):
    P = ctypes.c_void_p
    return (P * len(xs))(*[int(x) for x in xs])


def _shard_list(ts, name):
    if not isinstance(ts, (list, tuple)) or not ts:
        raise ValueError(f"{name} must be a non-empty list of tensors, one per shard")
    T, H, s = _rows(ts[0], f"{name}[0]")
    for j, t in enumerate(ts):
        _same(ts[0].device, ts[0].dtype, t, f"{name}[{j}]")
        Tj, Hj, sj = _rows(t, f"{name}[{j}]")
        if (Tj, Hj) != (T, H) or (T > 1 and sj != s):
            raise ValueError(f"{name}: every shard must have the same shape and row stride")
    return T, H, s


def _sums_all(t, name, P, T, dev):
    if t is None:
        return torch.empty((P, T), dtype=torch.float32, device=dev)
    if not (isinstance(t, torch.Tensor) and t.is_cuda and t.device == dev and t.dtype == torch.float32
            and t.is_contiguous() and tuple(t.shape) == (P, T)):
        raise ValueError(f"{name} must be a contiguous float32 CUDA tensor of shape [{P}, {T}]")
    return t


def qknorm_partial_stats_shards(q_shards, k_shards, q_sumsq_all=None, k_sumsq_all=None, *, stream=None,
                                launch: QknLaunch | dict | None = None):
    """Phase A local step for P shards of Q and of K in one launch: row p of
    the returned ``[P, T]`` float32 arrays ``(q_sumsq_all, k_sumsq_all)``
    holds the squared sums of shard p, exactly what P calls of
    ``qknorm_partial_stats`` would write."""
    P = len(q_shards)
    if len(k_shards) != P:
        raise ValueError("one K shard per Q shard")
    T, hq, sq = _shard_list(q_shards, "q_shards")
    Tk, hk, sk = _shard_list(k_shards, "k_shards")
    dev, dt = q_shards[0].device, q_shards[0].dtype
    _same(dev, dt, k_shards[0], "k_shards[0]")
    if T != Tk:
        raise ValueError("Q and K shards must have the same number of tokens")
    q_sumsq_all = _sums_all(q_sumsq_all, "q_sumsq_all", P, T, dev)
    k_sumsq_all = _sums_all(k_sumsq_all, "k_sumsq_all", P, T, dev)
    args = [P, _ptr_array([t.data_ptr() for t in q_shards]), sq, hq, q_sumsq_all.data_ptr(),
            _ptr_array([t.data_ptr() for t in k_shards]), sk, hk, k_sumsq_all.data_ptr(), T, _DTYPES[dt]]
    with _on(dev):
        s = _stream_handle(stream, dev)
        if launch is None:
            st = capi().qknorm_partial_stats_shards(*args, s)
        else:
            st = capi().qknorm_partial_stats_shards_launch(*args, s, ctypes.byref(_launch_struct(launch)))
    _clib.check(st, "qknorm_partial_stats_shards")
    return q_sumsq_all, k_sumsq_all


def qknorm_combine_apply_shards(q_in, k_in, gamma_q_shards, gamma_k_shards, q_sumsq_all: torch.Tensor,
                                k_sumsq_all: torch.Tensor, Hq_full: int, Hk_full: int, eps: float = 1e-6, *,
                                q_out=None, k_out=None, stream=None, launch: QknLaunch | dict | None = None):
    """Phase A aggregation and Phase B for P shards of Q and of K in one
    launch: the same results as P calls of ``qknorm_combine_apply`` with the
    same ``[P, T]`` partial sums.  Returns the lists ``(q_out, k_out)``."""
    P = len(q_in)
    if not (len(k_in) == len(gamma_q_shards) == len(gamma_k_shards) == P):
        raise ValueError("one K shard and one gamma slice of each tensor per Q shard")
    T, hq, sq = _shard_list(q_in, "q_in")
    Tk, hk, sk = _shard_list(k_in, "k_in")
    dev, dt = q_in[0].device, q_in[0].dtype
    _same(dev, dt, k_in[0], "k_in[0]")
    if T != Tk:
        raise ValueError("Q and K shards must have the same number of tokens")
    for t, name in ((q_sumsq_all, "q_sumsq_all"), (k_sumsq_all, "k_sumsq_all")):
        _sums_all(t, name, P, T, dev)
    if q_out is None:
        q_out = [_out_like(t, sq) for t in q_in]
    if k_out is None:
        k_out = [_out_like(t, sk) for t in k_in]
    if len(q_out) != P or len(k_out) != P:
        raise ValueError("one output per shard")
    for outs, name, (H, s) in ((q_out, "q_out", (hq, sq)), (k_out, "k_out", (hk, sk))):
        for j, t in enumerate(outs):
            _same(dev, dt, t, f"{name}[{j}]")
            To, Ho, so = _rows(t, f"{name}[{j}]")
            if (To, Ho) != (T, H) or (T > 1 and so != s):
                raise ValueError(f"{name}[{j}] must match its input's shape and row stride")
    gdt = gamma_dtype(dt)
    gq = [_vec(g, f"gamma_q_shards[{j}]", hq, gdt, dev) for j, g in enumerate(gamma_q_shards)]
    gk = [_vec(g, f"gamma_k_shards[{j}]", hk, gdt, dev) for j, g in enumerate(gamma_k_shards)]
    args = [P, _ptr_array([t.data_ptr() for t in q_in]), _ptr_array([t.data_ptr() for t in q_out]),
            _ptr_array(gq), sq, hq, q_sumsq_all.data_ptr(), int(Hq_full), _ptr_array([t.data_ptr() for t in k_in]),
            _ptr_array([t.data_ptr() for t in k_out]), _ptr_array(gk), sk, hk, k_sumsq_all.data_ptr(), int(Hk_full),
            T, float(eps), _DTYPES[dt]]
    with _on(dev):
        s = _stream_handle(stream, dev)
        if launch is None:
            st = capi().qknorm_combine_apply_shards(*args, s)
        else:
            st = capi().qknorm_combine_apply_shards_launch(*args, s, ctypes.byref(_launch_struct(launch)))
    _clib.check(st, "qknorm_combine_apply_shards")
    return q_out, k_out


# --------------------------------------------------------------------------- host planning (no GPU)

def plan_shape(rows: int, units_max: int, vectorized: bool, sm_count: int, elem_bytes: int = 2) -> dict:
    L = QknLaunch()
    st = capi().qknorm_plan_shape(rows, units_max, 1 if vectorized else 0, sm_count, elem_bytes,
                                  ctypes.byref(L))
    _clib.check(st, "qknorm_plan_shape")
    return L.as_dict()


def plan_grid(rows: int, blocks_per_sm: int, sm_count: int) -> int:
    return capi().qknorm_plan_grid(rows, blocks_per_sm, sm_count)


def regions_overlap(a: tuple, b: tuple) -> bool:
    """``a`` and ``b`` are ``(base, width_bytes, stride_bytes, rows)``."""
    return bool(capi().qknorm_regions_overlap(*a, *b))


from .host_pipeline import qknorm_layerwise_host, qknorm_packed_host  # noqa: E402  (uses qknorm_layerwise)
