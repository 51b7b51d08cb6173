"""ctypes loader for libgnorm.so (the C ABI declared in include/gnorm.h).

The shared library is built in-tree (``python gated_norm_b200/build.py``).  There is no
fallback: if the library is missing, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgnorm.so")

GNORM_OK = 0
GNORM_ERR_NULL = -1
GNORM_ERR_SHAPE = -2
GNORM_ERR_ALIGN = -3
GNORM_ERR_ALIAS = -4
GNORM_ERR_UNSUPPORTED = -5
GNORM_ERR_WORKSPACE = -6
GNORM_ERR_CUDA = -7
GNORM_ERR_ARG = -8
GNORM_N_MAX = 16384
GNORM_WORKSPACE_ALIGN = 256


class GnormPlan(ctypes.Structure):
    """Mirror of ``gnorm_plan`` in include/gnorm.h."""

    _fields_ = [
        ("kind", ctypes.c_int),
        ("threads_per_row", ctypes.c_int),
        ("chunks_per_thread", ctypes.c_int),
        ("consumer_threads", ctypes.c_int),
        ("rows_per_stage", ctypes.c_int),
        ("stages", ctypes.c_int),
        ("ctas_per_sm", ctypes.c_int),
        ("grid", ctypes.c_int),
        ("num_blocks", ctypes.c_int64),
        ("smem_bytes", ctypes.c_int),
        ("dynamic_schedule", ctypes.c_int),
        ("fused_reduce", ctypes.c_int),
        ("partials", ctypes.c_int),
        ("l2_prefetch", ctypes.c_int),
        ("direct_loads", ctypes.c_int),
    ]

    def as_dict(self) -> dict:
        return {name: getattr(self, name) for name, _ in self._fields_}


class GnormTuning(ctypes.Structure):
    """Mirror of ``gnorm_tuning`` in include/gnorm.h."""

    _fields_ = [(name, ctypes.c_int) for name in (
        "stage_bytes", "max_stages", "ctas_per_sm", "disable_pdl", "threads_per_row",
        "chunks_per_thread", "l2_prefetch", "tail_reduce", "chain_prefetch",
        "host_chunk_bytes", "fwd_direct", "bwd_direct", "fuse_fwd_bwd")]


class GnormFwdDesc(ctypes.Structure):
    """Mirror of ``gnorm_fwd_desc`` in include/gnorm.h."""

    _fields_ = [
        ("x", ctypes.c_void_p), ("ldx", ctypes.c_int64),
        ("g", ctypes.c_void_p), ("ldg", ctypes.c_int64),
        ("w", ctypes.c_void_p), ("w_fp32", ctypes.c_int),
        ("eps", ctypes.c_float),
        ("y", ctypes.c_void_p), ("ldy", ctypes.c_int64),
        ("rstd", ctypes.c_void_p),
        ("M", ctypes.c_int64), ("N", ctypes.c_int64),
    ]


class GnormBwdDesc(ctypes.Structure):
    """Mirror of ``gnorm_bwd_desc`` in include/gnorm.h."""

    _fields_ = [
        ("dy", ctypes.c_void_p), ("lddy", ctypes.c_int64),
        ("x", ctypes.c_void_p), ("ldx", ctypes.c_int64),
        ("g", ctypes.c_void_p), ("ldg", ctypes.c_int64),
        ("w", ctypes.c_void_p), ("w_fp32", ctypes.c_int),
        ("rstd", ctypes.c_void_p),
        ("dx", ctypes.c_void_p), ("lddx", ctypes.c_int64),
        ("dg", ctypes.c_void_p), ("lddg", ctypes.c_int64),
        ("dw", ctypes.c_void_p), ("dw_fp32", ctypes.c_int),
        ("deterministic", ctypes.c_int),
        ("M", ctypes.c_int64), ("N", ctypes.c_int64),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
    ]


_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int
_f32 = ctypes.c_float
_sz = ctypes.c_size_t

# name -> (restype, argtypes); every symbol include/gnorm.h declares.
SIGNATURES = {
    "gnorm_fwd": (_int, [_vp, _vp, _vp, _f32, _vp, _vp, _i64, _i64, _vp]),
    "gnorm_bwd": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _int, _int, _i64, _i64, _vp, _sz,
                         _vp]),
    "gnorm_bwd_noalloc": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _int, _int, _i64, _i64,
                                 _vp]),
    "gnorm_fwd_ex": (_int, [ctypes.POINTER(GnormFwdDesc), _vp]),
    "gnorm_bwd_ex": (_int, [ctypes.POINTER(GnormBwdDesc), _vp]),
    "gnorm_ckpt_step_ex": (_int, [ctypes.POINTER(GnormFwdDesc), ctypes.POINTER(GnormBwdDesc), _vp]),
    "gnorm_ckpt_step": (_int, [_vp, _vp, _vp, _f32, _vp, _vp, _vp, _vp, _vp, _vp, _int, _int, _i64,
                               _i64, _vp, _sz, _vp]),
    "gnorm_fwd_bwd_ex": (_int, [ctypes.POINTER(GnormFwdDesc), ctypes.POINTER(GnormBwdDesc), _vp]),
    "gnorm_fwd_bwd": (_int, [_vp, _vp, _vp, _f32, _vp, _vp, _vp, _vp, _vp, _vp, _int, _int, _i64,
                             _i64, _vp, _sz, _vp]),
    "gnorm_ckpt_step_host": (_int, [_vp, _vp, _vp, _f32, _vp, _vp, _vp, _vp, _vp, _vp, _int,
                                    _int, _i64, _i64, _vp, _sz, _vp]),
    "gnorm_ckpt_step_host_bytes": (_sz, [_i64, _i64, _int]),
    "gnorm_dw_reduce": (_int, [_vp, _i64, _i64, _vp, _int, _vp]),
    "gnorm_bwd_workspace_bytes": (_sz, [_i64, _i64, _int]),
    "gnorm_bwd_workspace_bytes_for": (_sz, [_i64, _i64, _int, _int]),
    "gnorm_status_string": (ctypes.c_char_p, [_int]),
    "gnorm_plan_query": (_int, [_int, _i64, _i64, _int, _int, _int, ctypes.POINTER(GnormPlan)]),
    "gnorm_device_error": (_int, [_int]),
    "gnorm_selftest_wait_timeout": (_int, [ctypes.c_uint, ctypes.POINTER(ctypes.c_ulonglong)]),
    "gnorm_set_tuning": (None, [ctypes.POINTER(GnormTuning)]),
    "gnorm_build_info": (ctypes.c_char_p, []),
}


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python gated_norm_b200/build.py` "
            "(the CUDA path has no CPU fallback)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = load()
