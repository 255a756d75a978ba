"""The C-ABI library loads, exports every entry point its header declares, and rejects
bad arguments on the host before touching a device.  No GPU needed: every call here
returns before its first CUDA runtime call."""

from __future__ import annotations

import ctypes
import glob
import os
import re

import pytest

from bwd_rmsnorm_fwd_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from bwd_rmsnorm_fwd_b200 import build
    build.build()
    return _lib.lib()


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^[A-Za-z_][\w\s\*]*?\b(rms_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_and_binding_agree(L):
    decl = declared_functions()
    assert len(decl) >= 11
    bound = sorted(n for n, _, _ in _lib.SIGNATURES)
    assert decl == bound
    for name in decl:
        assert hasattr(L, name), name


def test_exported_symbols_with_nm(L):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True,
                         text=True).stdout
    exported = set(re.findall(r"\bT (rms_\w+)", out))
    assert set(declared_functions()) <= exported


SH = _lib.shape(64, 1, 512)
A = 1 << 20  # fake, aligned device addresses: nothing below dereferences them


def rows(addr, st=512, sk=0):
    return _lib.rows(addr, st, sk)


def fwd(L, shape=SH, x=rows(A), w=A + (1 << 19), wdt=0, y=rows(A + (2 << 19)), rstd=A + (3 << 19)):
    return L.rms_train_fwd(shape, x, w, wdt, y, rstd, 1e-6, None)


def test_shape_errors(L):
    for bad in [_lib.shape(4, 1, 7), _lib.shape(4, 1, 0), _lib.shape(4, 0, 64),
                _lib.shape(-1, 1, 64), _lib.shape(4, 1, 8200), _lib.shape(1 << 30, 4, 64)]:
        assert fwd(L, shape=bad) == _lib.RMS_EINVAL
        assert L.rms_train_bwd_workspace_bytes(bad, 1, 0) == 0
        assert L.rms_train_bwd_path(bad, 1) == _lib.RMS_EINVAL
    assert b"H" in L.rms_last_error() or b"T" in L.rms_last_error()


def test_dtype_alignment_alias_errors(L):
    assert fwd(L, wdt=7) == _lib.RMS_EDTYPE
    assert fwd(L, x=rows(A + 8)) == _lib.RMS_EALIGN
    assert fwd(L, x=rows(A, st=516)) == _lib.RMS_EALIGN
    assert fwd(L, w=A + 4) == _lib.RMS_EALIGN
    assert fwd(L, rstd=A + 2) == _lib.RMS_EALIGN
    assert fwd(L, y=rows(A)) == _lib.RMS_EALIAS                  # y over x
    assert fwd(L, rstd=A + 128) == _lib.RMS_EALIAS               # rstd inside x
    assert fwd(L, y=rows(A + (2 << 19), st=256)) == _lib.RMS_EINVAL  # overlapping output rows
    assert fwd(L, x=rows(0)) == _lib.RMS_EINVAL


def test_backward_host_checks(L):
    x, dy, dx = rows(A), rows(A + (1 << 19)), rows(A + (2 << 19))
    w, rstd, dw = A + (3 << 19), A + (4 << 19), A + (5 << 19)
    ws = A + (8 << 19)
    need = L.rms_train_bwd_workspace_bytes(SH, 1, 0)
    assert need >= 256 + 512 * 8

    def bwd(**kw):
        a = dict(x=x, w=w, wdt=1, rstd=rstd, dy=dy, dx=dx, dw=dw, det=1, ws=ws, wsb=need, grid=0)
        a.update(kw)
        return L.rms_train_bwd(SH, a["x"], a["w"], a["wdt"], a["rstd"], a["dy"], a["dx"],
                               a["dw"], a["det"], a["ws"], a["wsb"], a["grid"], None)

    assert bwd(dw=w) == _lib.RMS_EALIAS                       # dw aliasing w
    assert bwd(dw=w + 16) == _lib.RMS_EALIAS
    assert bwd(dx=dy) == _lib.RMS_EALIAS
    assert bwd(ws=0) == _lib.RMS_EWORKSPACE
    assert bwd(wsb=need - 1) == _lib.RMS_EWORKSPACE
    assert bwd(ws=ws + 16) == _lib.RMS_EALIGN
    assert bwd(ws=A) == _lib.RMS_EALIAS                       # workspace over x
    assert bwd(grid=-1) == _lib.RMS_EINVAL
    assert bwd(grid=70000) == _lib.RMS_EINVAL
    assert bwd(wdt=3) == _lib.RMS_EDTYPE
    assert bwd(dw=dw + 4) == _lib.RMS_EALIGN
    assert bwd(rstd=0) == _lib.RMS_EINVAL


def test_plan_and_path_queries(L):
    b, l, s = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    for (T, heads, H), L_exp in [((131072, 1, 6144), 1), ((16384, 24, 256), 8),
                                 ((65537, 1, 1536), 4), ((4096, 1, 2048), 1), ((1000, 1, 512), 8),
                                 ((4096, 1, 3072), 2)]:
        sh = _lib.shape(T, heads, H)
        assert L.rms_det_plan(sh, ctypes.byref(b), ctypes.byref(l), ctypes.byref(s)) == 0
        assert l.value == L_exp and b.value in (8, 16, 32, 64) and s.value == 16
        R = T * heads
        chunks = -(-R // (b.value * l.value))
        # enough chunks for every SM, unless blocks are already at their minimum size
        assert R <= 2048 or chunks >= 148 or b.value == 8
    # small row counts take the single-launch program in both modes
    assert L.rms_train_bwd_path(_lib.shape(32, 1, 4096), 1) == 1
    assert L.rms_train_bwd_path(_lib.shape(32, 1, 4096), 0) == 1
    big = _lib.shape(131072, 1, 6144)
    assert L.rms_train_bwd_path(big, 1) == 2 and L.rms_train_bwd_path(big, 0) == 3
    # the deterministic workspace holds one FP64 row of H per chunk
    L.rms_det_plan(big, ctypes.byref(b), ctypes.byref(l), ctypes.byref(s))
    chunks = -(-131072 // (b.value * l.value))
    assert L.rms_train_bwd_workspace_bytes(big, 1, 0) >= chunks * 6144 * 8
    assert L.rms_train_bwd_workspace_bytes(big, 0, 0) < 1 << 20
    # the override moves the cut-over and restores
    prev = L.rms_set_small_rows_limit(0)
    assert L.rms_train_bwd_path(_lib.shape(32, 1, 4096), 1) == 2
    L.rms_set_small_rows_limit(prev)
    assert L.rms_train_bwd_path(_lib.shape(32, 1, 4096), 1) == 1
