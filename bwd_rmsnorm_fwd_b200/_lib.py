"""ctypes binding of librmsnorm_train.so (argument marshalling only).

The names and arguments mirror ``include/rmsnorm_train.h``.  Loading fails loudly
when the library has not been built: there is no fallback implementation.
"""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librmsnorm_train.so")

RMS_BF16 = 0
RMS_FP32 = 1

ERRORS = {
    0: "RMS_OK", -1: "RMS_EINVAL", -2: "RMS_EDTYPE", -3: "RMS_EALIGN", -4: "RMS_EALIAS",
    -5: "RMS_EWORKSPACE", -6: "RMS_ECUDA", -7: "RMS_ETIMEOUT",
}
RMS_OK, RMS_EINVAL, RMS_EDTYPE, RMS_EALIGN, RMS_EALIAS = 0, -1, -2, -3, -4
RMS_EWORKSPACE, RMS_ECUDA, RMS_ETIMEOUT = -5, -6, -7


class RmsRows(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("st", ctypes.c_int64), ("sk", ctypes.c_int64)]


class RmsShape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("heads", ctypes.c_int32), ("H", ctypes.c_int32)]


class RmsError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{ERRORS.get(code, code)}: {msg}")
        self.code = code


# (name, restype, argtypes) for every entry point of the header
_vp, _i32, _i64, _f32, _sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float,
                              ctypes.c_size_t)
SIGNATURES = [
    ("rms_train_fwd", _i32, [RmsShape, RmsRows, _vp, _i32, RmsRows, _vp, _f32, _vp]),
    ("rms_residual_train_fwd", _i32,
     [RmsShape, RmsRows, RmsRows, _vp, _i32, RmsRows, RmsRows, _vp, _f32, _vp]),
    ("rms_train_bwd", _i32,
     [RmsShape, RmsRows, _vp, _i32, _vp, RmsRows, RmsRows, _vp, _i32, _vp, _sz, _i32, _vp]),
    ("rms_residual_train_bwd", _i32,
     [RmsShape, RmsRows, _vp, _i32, _vp, RmsRows, RmsRows, RmsRows, _vp, _i32, _vp, _sz, _i32,
      _vp]),
    ("rms_train_bwd_accumulate", _i32,
     [RmsShape, RmsRows, _vp, _i32, _vp, RmsRows, RmsRows, _vp, _i32, _vp, _sz, _i32, _vp]),
    ("rms_residual_train_bwd_accumulate", _i32,
     [RmsShape, RmsRows, _vp, _i32, _vp, RmsRows, RmsRows, RmsRows, _vp, _i32, _vp, _sz, _i32,
      _vp]),
    ("rms_train_bwd_noalloc", _i32,
     [RmsShape, RmsRows, _vp, _i32, _vp, RmsRows, RmsRows, _vp, _vp]),
    ("rms_noalloc_status", _i32, [_vp]),
    ("rms_train_bwd_workspace_bytes", _sz, [RmsShape, _i32, _i32]),
    ("rms_det_plan", _i32, [RmsShape, ctypes.POINTER(ctypes.c_int32),
                            ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32)]),
    ("rms_det_shard_plan", _i32, [RmsShape, _i32, _i32, ctypes.POINTER(ctypes.c_int64),
                                  ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_size_t)]),
    ("rms_train_bwd_det_shard", _i32,
     [RmsShape, _i32, _i32, RmsRows, _vp, _i32, _vp, RmsRows, RmsRows, RmsRows, _vp, _vp, _sz,
      _i32, _vp]),
    ("rms_det_fold_segments", _i32, [RmsShape, _vp, _vp, _i32, _vp]),
    ("rms_train_bwd_path", _i32, [RmsShape, _i32]),
    ("rms_set_small_rows_limit", _i64, [_i64]),
    ("rms_set_l2_prefetch", _i32, [_i32]),
    ("rms_set_wait_limit_cycles", _i64, [_i64]),
    ("rms_status", _i32, [_vp, _vp]),
    ("rms_last_error", ctypes.c_char_p, []),
    ("rms_device_sms", _i32, []),
]

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it is missing (build it with
    ``python -m bwd_rmsnorm_fwd_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m bwd_rmsnorm_fwd_b200.build` (needs nvcc)")
        h = ctypes.CDLL(LIB_PATH)
        for name, res, args in SIGNATURES:
            f = getattr(h, name)
            f.restype = res
            f.argtypes = args
        _lib = h
    return _lib


def check(rc: int) -> None:
    if rc != RMS_OK:
        raise RmsError(rc, lib().rms_last_error().decode())


def shape(T: int, heads: int, H: int) -> RmsShape:
    return RmsShape(int(T), int(heads), int(H))


def rows(ptr: int, st: int, sk: int) -> RmsRows:
    return RmsRows(ctypes.c_void_p(int(ptr)), int(st), int(sk))
