"""ctypes prototypes for libqknorm.so (include/qknorm.h, include/qknorm_plan.h).

Loading fails loudly: there is no fallback of any kind.  Build the library
with ``python -m attention_normalization_b200.build``.
"""
from __future__ import annotations

import ctypes
import os

LIBRARY = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqknorm.so")

QKN_F32 = 0
QKN_BF16 = 1
QKN_F16 = 2
QKN_FP8_E4M3 = 3

QKN_OK = 0
QKN_ERR_INVALID_ARG = 1
QKN_ERR_MISALIGNED = 2  # reserved: never returned (unaligned buffers take a scalar-access kernel)
QKN_ERR_UNSUPPORTED = 3
QKN_ERR_CUDA = 4

QKN_KERNEL_REGISTER = 0
QKN_KERNEL_TWOPASS_VEC = 1
QKN_KERNEL_TWOPASS_SCALAR = 2


class QknLaunch(ctypes.Structure):
    """Mirror of ``qkn_launch``."""
    _fields_ = [("kernel", ctypes.c_int32), ("vec_per_thread", ctypes.c_int32),
                ("threads", ctypes.c_int32), ("grid", ctypes.c_int64)]

    def as_dict(self) -> dict:
        return {"kernel": self.kernel, "vec_per_thread": self.vec_per_thread,
                "threads": self.threads, "grid": self.grid}


class QknGemmSchedule(ctypes.Structure):
    """Mirror of ``qkn_gemm_schedule``."""
    _fields_ = [("clusters", ctypes.c_int32), ("units", ctypes.c_int32), ("group_units", ctypes.c_int32)]

    def as_dict(self) -> dict:
        return {f: getattr(self, f) for f, _ in self._fields_}


# Every symbol the headers declare, with (restype, argtypes).
_vp, _i64, _i32, _u64, _f32 = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32,
                               ctypes.c_uint64, ctypes.c_float)
_dt = ctypes.c_int
_st = ctypes.c_int
_LAYERWISE_ARGS = [_vp, _vp, _vp, _i64, _vp, _vp, _vp, _i64, _i64, _i32, _i32, _f32, _dt]
_HEADWISE_ARGS = [_vp, _vp, _vp, _i64, _i32, _vp, _vp, _vp, _i64, _i32, _i64, _i32, _f32, _dt]

PROTOTYPES = {
    "qknorm_qkv_gemm_schedule": (_st, [_i64, _i32, _i32, _i32, _i32, _i32, _i64, ctypes.POINTER(QknGemmSchedule)]),
    "qknorm_qkv_gemm_plan": (_st, [_i64, _i32, _i32, _i32, _i32, ctypes.POINTER(QknGemmSchedule)]),
    "qknorm_layerwise": (_st, _LAYERWISE_ARGS + [_vp]),
    "qknorm_partial_stats": (_st, [_vp, _i64, _i32, _vp, _vp, _i64, _i32, _vp, _i64, _dt, _vp]),
    "qknorm_headwise": (_st, _HEADWISE_ARGS + [_vp]),
    "qknorm_headwise_launch": (_st, _HEADWISE_ARGS + [_vp, ctypes.POINTER(QknLaunch)]),
    "qknorm_combine_apply": (_st, [_vp, _vp, _vp, _i64, _i32, _vp, _i32,
                                   _vp, _vp, _vp, _i64, _i32, _vp, _i32,
                                   _i32, _i64, _f32, _dt, _vp]),
    "qknorm_partial_stats_shards": (_st, [_i32, _vp, _i64, _i32, _vp, _vp, _i64, _i32, _vp, _i64, _dt, _vp]),
    "qknorm_combine_apply_shards": (_st, [_i32, _vp, _vp, _vp, _i64, _i32, _vp, _i32,
                                          _vp, _vp, _vp, _i64, _i32, _vp, _i32, _i64, _f32, _dt, _vp]),
    "qknorm_partial_stats_shards_launch": (_st, [_i32, _vp, _i64, _i32, _vp, _vp, _i64, _i32, _vp, _i64, _dt, _vp,
                                                 ctypes.POINTER(QknLaunch)]),
    "qknorm_combine_apply_shards_launch": (_st, [_i32, _vp, _vp, _vp, _i64, _i32, _vp, _i32,
                                                 _vp, _vp, _vp, _i64, _i32, _vp, _i32, _i64, _f32, _dt, _vp,
                                                 ctypes.POINTER(QknLaunch)]),
    "qknorm_status_string": (ctypes.c_char_p, [_st]),
    "qknorm_qkv_gemm_stats": (_st, [_vp, _i64, _vp, _i64, _vp, _i64, _i64, _i32, _i32, _i32, _i32,
                                    _vp, _vp, _dt, _vp]),
    "qknorm_qkv_projection_workspace_bytes": (_i64, [_i64, _i32, _i32]),
    "qknorm_qkv_projection": (_st, [_vp, _i64, _vp, _i64, _vp, _i64, _vp, _vp, _i64, _i32, _i32, _i32, _i32,
                                    _f32, _vp, _i64, _dt, _vp]),
    "qknorm_device_timeouts": (_st, [ctypes.POINTER(ctypes.c_int32)]),
    "qknorm_qkv_projection_noalloc": (_st, [_vp, _i64, _vp, _i64, _vp, _i64, _vp, _vp, _i64, _i32, _i32, _i32,
                                            _i32, _f32, _dt, _vp]),
    "qknorm_qkv_projection_noalloc_max_bytes": (_i64, []),
    "qknorm_tp_recv_bytes": (_i64, [_i32, _i64]),
    "qknorm_tp_layerwise": (_st, [_i32, _i32, _i32, _vp, _vp, _vp, _i64, _i32, _i32, _vp, _vp, _vp, _i64, _i32, _i32,
                                  _i64, _f32, _dt, _vp, ctypes.c_uint32, _i32, _u64, _vp]),
    "qknorm_tp_layerwise_scope": (_st, [_i32, _i32, _i32, _vp, _vp, _vp, _i64, _i32, _i32, _vp, _vp, _vp, _i64, _i32,
                                        _i32, _i64, _f32, _dt, _vp, ctypes.c_uint32, _i32, _u64, _i32, _vp]),
    "qknorm_layerwise_host": (_st, _LAYERWISE_ARGS + [_vp, _i64, _i64, _vp, _vp, _vp]),
    "qknorm_layerwise_host_ring_bytes": (_i64, [_i64, _i32, _i32, _dt, _i32]),
    "qknorm_last_error": (ctypes.c_char_p, []),
    "qknorm_version": (ctypes.c_int, []),
    "qknorm_register_max_threads": (_i32, [_i32]),
    "qknorm_plan_shape": (_st, [_i64, _i64, _i32, _i32, _i32, ctypes.POINTER(QknLaunch)]),
    "qknorm_plan_grid": (_i64, [_i64, _i32, _i32]),
    "qknorm_regions_overlap": (ctypes.c_int, [_u64, _i64, _i64, _i64, _u64, _i64, _i64, _i64]),
    "qknorm_layerwise_plan": (_st, _LAYERWISE_ARGS + [ctypes.POINTER(QknLaunch)]),
    "qknorm_layerwise_launch": (_st, _LAYERWISE_ARGS + [_vp, ctypes.POINTER(QknLaunch)]),
    "qknorm_partial_stats_launch": (_st, [_vp, _i64, _i32, _vp, _vp, _i64, _i32, _vp, _i64, _dt, _vp,
                                          ctypes.POINTER(QknLaunch)]),
    "qknorm_combine_apply_launch": (_st, [_vp, _vp, _vp, _i64, _i32, _vp, _i32,
                                          _vp, _vp, _vp, _i64, _i32, _vp, _i32,
                                          _i32, _i64, _f32, _dt, _vp, ctypes.POINTER(QknLaunch)]),
}

_lib = None


def load() -> ctypes.CDLL:
    """Load libqknorm.so (once) and attach the prototypes."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIBRARY):
        raise RuntimeError(
            f"libqknorm.so is not built ({LIBRARY} missing). Build it with "
            "`python -m attention_normalization_b200.build`; there is no fallback path.")
    lib = ctypes.CDLL(LIBRARY)
    for name, (restype, argtypes) in PROTOTYPES.items():
        fn = getattr(lib, name)
        fn.restype = restype
        fn.argtypes = argtypes
    _lib = lib
    return lib


class QKNormError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = load()
        msg = lib.qknorm_last_error().decode(errors="replace")
        name = lib.qknorm_status_string(status).decode()
        super().__init__(f"{where}: {name} ({status}): {msg}")
        self.status = status


def check(status: int, where: str) -> None:
    if status != QKN_OK:
        raise QKNormError(status, where)
