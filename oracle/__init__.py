"""Oracle for training RMSNorm -- TEST INFRASTRUCTURE ONLY.

A plain FP64 CPU definition of what the CUDA path computes (see
``rmsnorm_oracle.cpp`` for the definitions and the passages they follow).  Only
``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package.  The product library neither imports nor links it, and
the two share no code.

Arrays: row tensors are dense ``[R, H]`` numpy ``uint16`` arrays of BF16 bits;
the weight is ``uint16`` BF16 bits or ``float32``; rstd is ``float32 [R]``.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rmsnorm_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (C++17, -O2, no fast-math) into ``liboracle.so``."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["g++", "-std=c++17", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC",
             "-shared", "-pthread", _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB)
    i64, i32, vp, f32, f64 = (ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_float,
                              ctypes.c_double)
    lib.oracle_bf16_from_f64.argtypes = [i64, vp, vp]
    lib.oracle_f64_from_bf16.argtypes = [i64, vp, vp]
    lib.oracle_fwd_f64.argtypes = [i64, i64, vp, vp, f64, vp, vp, i32]
    lib.oracle_bwd_f64.argtypes = [i64, i64, vp, vp, vp, vp, vp, vp, vp, i32]
    lib.oracle_train_fwd.argtypes = [i64, i64, vp, vp, vp, i32, f32, vp, vp, vp, vp, i32]
    lib.oracle_train_bwd.argtypes = [i64, i64, vp, vp, i32, vp, vp, vp, vp, vp, i32]
    lib.oracle_hardware_threads.restype = i32
    for f in ("oracle_bf16_from_f64", "oracle_f64_from_bf16", "oracle_fwd_f64",
              "oracle_bwd_f64", "oracle_train_fwd", "oracle_train_bwd"):
        getattr(lib, f).restype = None
    _lib = lib
    return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def hardware_threads() -> int:
    return int(_load().oracle_hardware_threads())


# ---- conversions ------------------------------------------------------------------------

def bf16_from_f64(v) -> np.ndarray:
    """Round doubles to BF16 bits, nearest-even, in one step."""
    v = _c(v, np.float64)
    out = np.empty(v.shape, np.uint16)
    _load().oracle_bf16_from_f64(v.size, _ptr(v), _ptr(out))
    return out


def f64_from_bf16(b) -> np.ndarray:
    b = _c(b, np.uint16)
    out = np.empty(b.shape, np.float64)
    _load().oracle_f64_from_bf16(b.size, _ptr(b), _ptr(out))
    return out


# ---- FP64 definitions on double arrays -----------------------------------------------------

def fwd_f64(x, w, eps: float, nthreads: int = 0):
    """Unrounded forward: returns (y64 [R,H], rstd64 [R])."""
    x = _c(x, np.float64)
    w = _c(w, np.float64)
    R, H = x.shape
    y = np.empty((R, H), np.float64)
    rstd = np.empty(R, np.float64)
    _load().oracle_fwd_f64(R, H, _ptr(x), _ptr(w), float(eps), _ptr(y), _ptr(rstd), nthreads)
    return y, rstd


def bwd_f64(x, w, rstd, dy, dh=None, nthreads: int = 0):
    """Unrounded backward: returns (dx64 [R,H], dw64 [H])."""
    x = _c(x, np.float64)
    w = _c(w, np.float64)
    rstd = _c(rstd, np.float64)
    dy = _c(dy, np.float64)
    dh = None if dh is None else _c(dh, np.float64)
    R, H = x.shape
    dx = np.empty((R, H), np.float64)
    dw = np.empty(H, np.float64)
    _load().oracle_bwd_f64(R, H, _ptr(x), _ptr(w), _ptr(rstd), _ptr(dy), _ptr(dh), _ptr(dx),
                           _ptr(dw), nthreads)
    return dx, dw


# ---- the API-level oracle ------------------------------------------------------------------

def _weight(w):
    if w.dtype == np.uint16:
        return _c(w, np.uint16), 0
    if w.dtype == np.float32:
        return _c(w, np.float32), 1
    raise TypeError("weight must be uint16 (BF16 bits) or float32")


def train_fwd(x, w, eps: float = 1e-6, residual=None, nthreads: int = 0, want_rstd64=False):
    """Forward on BF16 bits.  Returns (y, rstd) or, with a residual, (h, y, rstd);
    with ``want_rstd64`` the unrounded rstd is appended."""
    x = _c(x, np.uint16)
    R, H = x.shape
    res = None if residual is None else _c(residual, np.uint16)
    w, w_dt = _weight(w)
    y = np.empty((R, H), np.uint16)
    h = np.empty((R, H), np.uint16) if res is not None else None
    rstd = np.empty(R, np.float32)
    rstd64 = np.empty(R, np.float64) if want_rstd64 else None
    _load().oracle_train_fwd(R, H, _ptr(x), _ptr(res), _ptr(w), w_dt, float(eps), _ptr(h),
                             _ptr(y), _ptr(rstd), _ptr(rstd64), nthreads)
    out = (y, rstd) if res is None else (h, y, rstd)
    return out + (rstd64,) if want_rstd64 else out


def train_bwd(x, w, rstd, dy, dh=None, nthreads: int = 0, want_dx=True, want_dw=True):
    """Backward on BF16 bits with the caller's FP32 rstd.  ``x`` is h in the residual
    form.  Returns (dx BF16 bits or None, dw64 or None); dx is grad_h when dh is given."""
    x = _c(x, np.uint16)
    R, H = x.shape
    w, w_dt = _weight(w)
    rstd = _c(rstd, np.float32)
    dy = _c(dy, np.uint16)
    dh = None if dh is None else _c(dh, np.uint16)
    dx = np.empty((R, H), np.uint16) if want_dx else None
    dw = np.empty(H, np.float64) if want_dw else None
    _load().oracle_train_bwd(R, H, _ptr(x), _ptr(w), w_dt, _ptr(rstd), _ptr(dy), _ptr(dh),
                             _ptr(dx), _ptr(dw), nthreads)
    return dx, dw
