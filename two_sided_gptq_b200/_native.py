"""ctypes binding of ``libbakron.so`` (declarations mirror ``include/bakron.h``).

Loading fails loudly: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import enum
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbakron.so")


class Status(enum.IntEnum):
    OK = 0
    ERR_INVALID_ARG = 1
    ERR_ALIGNMENT = 2
    ERR_NOT_SPD = 3
    ERR_NONFINITE = 4
    ERR_DEVICE_TIMEOUT = 5
    ERR_CUDA = 6
    ERR_WORKSPACE = 7
    ERR_BAD_FACTOR = 8


class BakronError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = Status(status)
        msg = _lib.bakron_status_string(int(status)).decode() if _lib is not None else str(status)
        super().__init__(f"{where}: {self.status.name} ({msg})" if where else f"{self.status.name} ({msg})")


class Quantizer(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int32), ("qmin", ctypes.c_int32), ("qmax", ctypes.c_int32),
                ("row_scale", ctypes.c_void_p), ("shrink_grid", ctypes.c_int32)]


class BatchItem(ctypes.Structure):
    _fields_ = [("W", ctypes.c_void_p), ("m", ctypes.c_int64), ("n", ctypes.c_int64), ("LA", ctypes.c_void_p),
                ("LB", ctypes.c_void_p), ("V", ctypes.c_void_p), ("codes", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("ws", ctypes.c_void_p), ("ws_bytes", ctypes.c_size_t)]


class Config(ctypes.Structure):
    _fields_ = [("tile", ctypes.c_int32), ("gemm", ctypes.c_int32), ("use_graph", ctypes.c_int32),
                ("timeout_ms", ctypes.c_int32), ("wt_out", ctypes.c_void_p), ("profile", ctypes.c_int32),
                ("leaf", ctypes.c_int32), ("b_identity", ctypes.c_int32), ("fuse_width", ctypes.c_int32),
                ("self_test_omit", ctypes.c_int32)]


class Profile(ctypes.Structure):
    _fields_ = [("prep_ms", ctypes.c_double), ("leaf_ms", ctypes.c_double), ("stage1_ms", ctypes.c_double),
                ("stage2_ms", ctypes.c_double), ("total_ms", ctypes.c_double),
                ("prep_launches", ctypes.c_int64), ("leaf_launches", ctypes.c_int64),
                ("stage1_launches", ctypes.c_int64), ("stage2_launches", ctypes.c_int64),
                ("fused_ms", ctypes.c_double), ("fused_launches", ctypes.c_int64)]


class PlanStats(ctypes.Structure):
    _fields_ = [("tiles_m", ctypes.c_int64), ("tiles_n", ctypes.c_int64), ("tile_diagonals", ctypes.c_int64),
                ("nodes", ctypes.c_int64), ("leaves", ctypes.c_int64), ("update_flops", ctypes.c_double),
                ("stage1_flops", ctypes.c_double), ("stage2_flops", ctypes.c_double),
                ("structural_flops", ctypes.c_double), ("leaf_update_flops", ctypes.c_double)]


# name -> (restype, argtypes); every function declared in include/bakron.h
_vp, _i64, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
class ProfileLaunch(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("k", ctypes.c_int32), ("h", ctypes.c_int32), ("l", ctypes.c_int32),
                ("ms", ctypes.c_double), ("flops", ctypes.c_double), ("structural_flops", ctypes.c_double)]


SIGNATURES = {
    "bakron_factor_workspace_size": (_sz, [_i64, _i64]),
    "bakron_factor": (ctypes.c_int, [_vp, _i64, _vp, _i64, _vp, _vp, _vp, _sz, _vp]),
    "bakron_solve_workspace_size": (_sz, [_i64, _i64, ctypes.POINTER(Config)]),
    "bakron_solve": (ctypes.c_int, [_vp, _i64, _i64, _vp, _vp, ctypes.POINTER(Quantizer), _vp, _vp, _vp, _vp, _sz,
                                    ctypes.POINTER(Config), _vp]),
    "bakron_solve_host_workspace_size": (_sz, [_i64, _i64, ctypes.POINTER(Config)]),
    "bakron_solve_host": (ctypes.c_int, [_vp, _i64, _i64, _vp, _vp, ctypes.POINTER(Quantizer), _vp, _vp, _vp, _vp,
                                         _sz, ctypes.POINTER(Config), _vp]),
    "bakron_proxy_loss_workspace_size": (_sz, [_i64, _i64]),
    "bakron_proxy_loss": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _i64, _vp, ctypes.POINTER(ctypes.c_double), _vp,
                                         _sz, _vp]),
    "bakron_get_status": (ctypes.c_int, [_vp, _sz, _vp]),
    "bakron_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_int32, _vp, _sz, _vp]),
    "bakron_selftest_band_abort_workspace_size": (_sz, []),
    "bakron_selftest_band_abort": (ctypes.c_int, [ctypes.c_int32, _vp, _sz, _vp]),
    "bakron_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "bakron_plan_stats": (ctypes.c_int, [_i64, _i64, ctypes.POINTER(Config), ctypes.POINTER(PlanStats)]),
    "bakron_version": (ctypes.c_char_p, []),
    "bakron_get_profile": (ctypes.c_int, [ctypes.POINTER(Profile)]),
    "bakron_get_profile_launches": (_i64, [ctypes.POINTER(ProfileLaunch), _i64]),
    "bakron_gram_workspace_size": (_sz, [_i64, _i64]),
    "bakron_gram": (ctypes.c_int, [_vp, _i64, _i64, ctypes.c_float, _vp, _vp, _sz, _vp]),
    "bakron_solve_batch": (ctypes.c_int, [ctypes.POINTER(BatchItem), ctypes.c_int32, ctypes.POINTER(Quantizer),
                                          ctypes.POINTER(Config), ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32]),
    "bakron_tune_leaf": (ctypes.c_int, [_vp, _i64, _i64, _vp, _vp, ctypes.POINTER(Quantizer), _vp, _vp, _vp, _vp, _sz,
                                        ctypes.POINTER(Config), _vp, ctypes.POINTER(ctypes.c_int32),
                                        ctypes.POINTER(ctypes.c_double)]),
    "bakron_solve_noalloc": (ctypes.c_int, [_vp, _i64, _i64, _vp, _vp, ctypes.POINTER(Quantizer), _vp, _vp, _vp,
                                            ctypes.POINTER(Config), _vp, ctypes.POINTER(ctypes.c_int32)]),
}

_lib = None


def load(path: str | None = None):
    """Load ``libbakron.so`` (raises if it is missing: build it with
    ``python -m two_sided_gptq_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise ImportError(f"libbakron.so not found at {p}; build it with `python -m two_sided_gptq_b200.build`")
    lib = ctypes.CDLL(p)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def check(status: int, where: str = ""):
    if status != 0:
        raise BakronError(status, where)
