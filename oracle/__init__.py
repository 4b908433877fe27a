"""CPU oracle for layerwise QK-RMSNorm — TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It never imports the CUDA package and
the CUDA package never imports it; the two share no code.

This module only marshals numpy arrays into the plain C oracle
(``qknorm_oracle.c``), which computes in double precision:

* ``rmsnorm_rows``   — RMS-Norm over full rows (Background, Equation 1 of
  "SwiftQK: Fast and Communication-Efficient Tensor Parallelism for Query-Key
  Normalization"); the FP64 gold of Fig. 2(b).
* ``rmsnorm_heads``  — headwise RMS-Norm (one factor per attention head, the
  other granularity the Background section names), gamma shared by the heads.
* ``partial_sumsq``  — Phase A's per-shard squared sum.
* ``combine_apply``  — Phase A's aggregation of the shard sums, then Phase B's
  weight multiplication and global RMS scaling of one shard.
* ``project_rows``   — the linear projection that produces Q, K and V
  (Background: Pre-LN layers), in double, rounded once to the element type.
* ``bf16_decode`` / ``bf16_encode`` — the element codec.

Arrays: fp32 data is passed as ``np.float32``, IEEE half as ``np.float16``,
bfloat16 as its raw bit patterns in ``np.uint16`` and FP8 E4M3 ("fn") as its
raw bit patterns in ``np.uint8`` (with E4M3 data, gamma is bfloat16 bits).  A 2-D input ``x`` of shape ``(T, stride)``
(or any C-contiguous array whose rows are ``stride`` elements apart) holds row
``t`` at element ``t * stride``; only its first ``H`` columns are read.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

F32 = 0
BF16 = 1
F16 = 2
E4M3 = 3

_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    # A test may point this at a deliberately broken build of the oracle to
    # check that the pins catch the mistake.
    path = os.environ.get("QKNORM_ORACLE_LIB") or _build.build()
    lib = ctypes.CDLL(path)
    vp, i64, i32, dbl = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_double
    lib.oracle_version.restype = ctypes.c_int
    lib.oracle_bf16_decode.argtypes = [ctypes.c_uint16]
    lib.oracle_bf16_decode.restype = dbl
    lib.oracle_bf16_encode_rne.argtypes = [dbl]
    lib.oracle_bf16_encode_rne.restype = ctypes.c_uint16
    lib.oracle_f16_decode.argtypes = [ctypes.c_uint16]
    lib.oracle_f16_decode.restype = dbl
    lib.oracle_f16_encode_rne.argtypes = [dbl]
    lib.oracle_f16_encode_rne.restype = ctypes.c_uint16
    lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_decode.restype = dbl
    lib.oracle_e4m3_encode_rne_sat.argtypes = [dbl]
    lib.oracle_e4m3_encode_rne_sat.restype = ctypes.c_uint8
    lib.oracle_rmsnorm_rows.argtypes = [vp, i64, i64, i32, vp, dbl, ctypes.c_int,
                                        vp, i64, vp, vp]
    lib.oracle_rmsnorm_rows.restype = ctypes.c_int
    lib.oracle_qknorm_layerwise.argtypes = [vp, i64, vp, i32, vp, i64, vp, i32,
                                            i64, dbl, ctypes.c_int, vp, vp]
    lib.oracle_qknorm_layerwise.restype = ctypes.c_int
    lib.oracle_rmsnorm_heads.argtypes = [vp, i64, i64, i32, i32, vp, dbl, ctypes.c_int, vp, vp]
    lib.oracle_project_rows.argtypes = [vp, i64, vp, i64, i64, i32, vp, i64, i32, ctypes.c_int, vp, vp]
    lib.oracle_project_rows.restype = ctypes.c_int
    lib.oracle_rmsnorm_heads.restype = ctypes.c_int
    lib.oracle_partial_sumsq.argtypes = [vp, i64, i64, i32, ctypes.c_int, vp]
    lib.oracle_partial_sumsq.restype = ctypes.c_int
    lib.oracle_combine_apply.argtypes = [vp, i64, i64, i32, vp, vp, i32, i32, dbl,
                                         ctypes.c_int, vp, i64, vp]
    lib.oracle_combine_apply.restype = ctypes.c_int
    _lib = lib
    return lib


def _dtype_code(arr: np.ndarray) -> int:
    if arr.dtype == np.float32:
        return F32
    if arr.dtype == np.uint16:
        return BF16
    if arr.dtype == np.float16:
        return F16
    if arr.dtype == np.uint8:
        return E4M3
    raise TypeError(f"oracle takes float32, float16, uint16 (bfloat16 bits) or uint8 (E4M3 bits), "
                    f"got {arr.dtype}")


def _gamma_dtype(x_dtype):
    """gamma has the element type of x, except bfloat16 bits with E4M3 data."""
    return np.dtype(np.uint16) if x_dtype == np.uint8 else x_dtype


def _ptr(arr):
    return None if arr is None else arr.ctypes.data


def _check_rows(x: np.ndarray, stride: int, T: int, H: int):
    if not x.flags.c_contiguous:
        raise ValueError("oracle input must be C-contiguous")
    if T > 0 and x.size < (T - 1) * stride + H:
        raise ValueError("input too small for T rows of the given stride")


def bf16_decode(bits) -> np.ndarray:
    lib = _load()
    b = np.asarray(bits, dtype=np.uint16)
    return np.array([lib.oracle_bf16_decode(int(v)) for v in b.ravel()],
                    dtype=np.float64).reshape(b.shape)


def bf16_encode(values) -> np.ndarray:
    lib = _load()
    v = np.asarray(values, dtype=np.float64)
    return np.array([lib.oracle_bf16_encode_rne(float(a)) for a in v.ravel()],
                    dtype=np.uint16).reshape(v.shape)


def f16_decode(bits) -> np.ndarray:
    lib = _load()
    b = np.asarray(bits, dtype=np.uint16)
    return np.array([lib.oracle_f16_decode(int(v)) for v in b.ravel()], dtype=np.float64).reshape(b.shape)


def f16_encode(values) -> np.ndarray:
    """Bit patterns (uint16) of the IEEE half values nearest to `values`."""
    lib = _load()
    v = np.asarray(values, dtype=np.float64)
    return np.array([lib.oracle_f16_encode_rne(float(a)) for a in v.ravel()], dtype=np.uint16).reshape(v.shape)


def e4m3_decode(bits) -> np.ndarray:
    lib = _load()
    b = np.asarray(bits, dtype=np.uint8)
    return np.array([lib.oracle_e4m3_decode(int(v)) for v in b.ravel()], dtype=np.float64).reshape(b.shape)


def e4m3_encode(values) -> np.ndarray:
    lib = _load()
    v = np.asarray(values, dtype=np.float64)
    return np.array([lib.oracle_e4m3_encode_rne_sat(float(a)) for a in v.ravel()], dtype=np.uint8).reshape(v.shape)


def rmsnorm_rows(x: np.ndarray, H: int, gamma: np.ndarray, eps: float,
                 stride: int | None = None, T: int | None = None):
    """RMS-Norm of rows of width ``H``.

    Returns ``(y, y_exact, sumsq)``: ``y`` has the input's element type with
    shape ``(T, H)``, ``y_exact`` is the unrounded float64 result ``(T, H)``,
    ``sumsq`` the float64 squared sums ``(T,)``.
    """
    lib = _load()
    dt = _dtype_code(x)
    if stride is None:
        stride = x.shape[-1]
    if T is None:
        T = x.size // stride if x.ndim == 1 else int(np.prod(x.shape[:-1])) * x.shape[-1] // stride
    _check_rows(x, stride, T, H)
    g = np.ascontiguousarray(gamma)
    if g.dtype != _gamma_dtype(x.dtype) or g.size < H:
        raise ValueError("gamma must have the gamma type of the input and at least H elements")
    y = np.zeros((T, H), dtype=x.dtype)
    y_exact = np.zeros((T, H), dtype=np.float64)
    sumsq = np.zeros((T,), dtype=np.float64)
    st = lib.oracle_rmsnorm_rows(_ptr(x), stride, T, H, _ptr(g), float(eps), dt,
                                 _ptr(y), H, _ptr(y_exact), _ptr(sumsq))
    if st != 0:
        raise ValueError(f"oracle_rmsnorm_rows rejected its arguments (status {st})")
    return y, y_exact, sumsq


def qknorm_layerwise(q: np.ndarray, q_stride: int, gamma_q: np.ndarray, Hq: int,
                     k: np.ndarray, k_stride: int, gamma_k: np.ndarray, Hk: int,
                     T: int, eps: float):
    """Layerwise QK-Norm of one batch; returns contiguous ``(q_out, k_out)``."""
    lib = _load()
    dt = _dtype_code(q)
    if _dtype_code(k) != dt:
        raise TypeError("q and k must share an element type")
    _check_rows(q, q_stride, T, Hq)
    _check_rows(k, k_stride, T, Hk)
    gq = np.ascontiguousarray(gamma_q)
    gk = np.ascontiguousarray(gamma_k)
    q_out = np.zeros((T, Hq), dtype=q.dtype)
    k_out = np.zeros((T, Hk), dtype=k.dtype)
    st = lib.oracle_qknorm_layerwise(_ptr(q), q_stride, _ptr(gq), Hq, _ptr(k), k_stride,
                                     _ptr(gk), Hk, T, float(eps), dt, _ptr(q_out), _ptr(k_out))
    if st != 0:
        raise ValueError(f"oracle_qknorm_layerwise rejected its arguments (status {st})")
    return q_out, k_out


def rmsnorm_heads(x: np.ndarray, n_heads: int, head_dim: int, gamma: np.ndarray, eps: float,
                  stride: int, T: int):
    """Headwise RMS-Norm: each of the n_heads heads of head_dim elements in a
    row is normalized on its own with the shared gamma [head_dim].  Returns
    ``(y, y_exact)`` of shape ``(T, n_heads * head_dim)``."""
    lib = _load()
    dt = _dtype_code(x)
    W = n_heads * head_dim
    _check_rows(x, stride, T, W)
    g = np.ascontiguousarray(gamma)
    if g.dtype != _gamma_dtype(x.dtype) or g.size < head_dim:
        raise ValueError("gamma must have the gamma type of the input and head_dim elements")
    y = np.zeros((T, W), dtype=x.dtype)
    y_exact = np.zeros((T, W), dtype=np.float64)
    st = lib.oracle_rmsnorm_heads(_ptr(x), stride, T, n_heads, head_dim, _ptr(g), float(eps), dt,
                                  _ptr(y), _ptr(y_exact))
    if st != 0:
        raise ValueError(f"oracle_rmsnorm_heads rejected its arguments (status {st})")
    return y, y_exact


def partial_sumsq(x: np.ndarray, h_shard: int, stride: int, T: int) -> np.ndarray:
    """Phase A local step: float64 squared sum of each row's first ``h_shard`` columns."""
    lib = _load()
    dt = _dtype_code(x)
    _check_rows(x, stride, T, h_shard)
    out = np.zeros((T,), dtype=np.float64)
    st = lib.oracle_partial_sumsq(_ptr(x), stride, T, h_shard, dt, _ptr(out))
    if st != 0:
        raise ValueError(f"oracle_partial_sumsq rejected its arguments (status {st})")
    return out


def combine_apply(x: np.ndarray, h_shard: int, stride: int, T: int, gamma_shard: np.ndarray,
                  sumsq_all: np.ndarray, H_full: int, eps: float):
    """Aggregate ``sumsq_all`` (shape ``(P, T)``, float64) in order p = 0..P-1,
    then scale this shard: returns ``(y, y_exact)`` of shape ``(T, h_shard)``."""
    lib = _load()
    dt = _dtype_code(x)
    _check_rows(x, stride, T, h_shard)
    s = np.ascontiguousarray(sumsq_all, dtype=np.float64)
    if s.ndim != 2 or s.shape[1] != T:
        raise ValueError("sumsq_all must have shape (P, T)")
    g = np.ascontiguousarray(gamma_shard)
    y = np.zeros((T, h_shard), dtype=x.dtype)
    y_exact = np.zeros((T, h_shard), dtype=np.float64)
    st = lib.oracle_combine_apply(_ptr(x), stride, T, h_shard, _ptr(g), _ptr(s), s.shape[0],
                                  H_full, float(eps), dt, _ptr(y), h_shard, _ptr(y_exact))
    if st != 0:
        raise ValueError(f"oracle_combine_apply rejected its arguments (status {st})")
    return y, y_exact


def project_rows(x: np.ndarray, w: np.ndarray, rows, D: int | None = None, N: int | None = None,
                 x_stride: int | None = None, w_stride: int | None = None):
    """The linear projection ``y[i][n] = sum_d x[rows[i]][d] * w[n][d]`` in
    double, W stored ``[N][D]`` (one row per output column).

    ``x`` is ``(T, x_stride)`` and ``w`` ``(N, w_stride)``, both of one element
    type; only the first ``D`` columns are read.  Returns ``(y, y_exact)``:
    ``y`` ``(n_rows, N)`` rounded once to the element type, ``y_exact`` the
    float64 sums.
    """
    lib = _load()
    dt = _dtype_code(x)
    if _dtype_code(w) != dt:
        raise TypeError("x and w must share an element type")
    if x.ndim != 2 or w.ndim != 2:
        raise ValueError("x and w must be 2-D")
    x_stride = x.shape[1] if x_stride is None else x_stride
    w_stride = w.shape[1] if w_stride is None else w_stride
    D = x_stride if D is None else D
    N = w.shape[0] if N is None else N
    if not (x.flags.c_contiguous and w.flags.c_contiguous):
        raise ValueError("oracle inputs must be C-contiguous")
    if w.size < (N - 1) * w_stride + D:
        raise ValueError("w too small for N rows of the given stride")
    T = x.size // x_stride
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).ravel())
    y = np.zeros((r.size, N), dtype=x.dtype)
    y_exact = np.zeros((r.size, N), dtype=np.float64)
    st = lib.oracle_project_rows(_ptr(x), x_stride, _ptr(r), r.size, T, D, _ptr(w), w_stride, N, dt,
                                 _ptr(y), _ptr(y_exact))
    if st != 0:
        raise ValueError(f"oracle_project_rows rejected its arguments (status {st})")
    return y, y_exact


def version() -> int:
    return _load().oracle_version()


__all__ = ["F32", "BF16", "F16", "E4M3", "bf16_decode", "bf16_encode", "f16_decode", "f16_encode",
           "e4m3_decode", "e4m3_encode", "rmsnorm_rows", "rmsnorm_heads", "qknorm_layerwise", "partial_sumsq",
           "combine_apply", "project_rows", "version"]
