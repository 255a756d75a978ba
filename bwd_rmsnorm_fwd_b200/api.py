"""Torch-facing wrappers over the C ABI.

PyTorch provides device memory and the current stream; every step of the
computation runs in librmsnorm_train's kernels.  Row tensors are BF16 CUDA tensors
shaped ``[T, H]`` or ``[T, heads, H]`` with unit innermost stride (any token/head
strides that are multiples of 8 elements).  Outputs are allocated with the input's
strides.
"""

from __future__ import annotations

import torch

from . import _lib

__all__ = [
    "rmsnorm_train_fwd", "rmsnorm_train_bwd", "Workspace", "det_plan", "bwd_path",
    "set_small_rows_limit", "status", "forward_status",
]


def _view(t: torch.Tensor, name: str):
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16 (got {t.dtype})")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dim() == 2:
        T, H = t.shape
        heads, st, sk = 1, t.stride(0), 0
    elif t.dim() == 3:
        T, heads, H = t.shape
        st, sk = t.stride(0), t.stride(1)
    else:
        raise ValueError(f"{name} must be [T, H] or [T, heads, H]")
    if H > 0 and t.stride(-1) != 1:
        raise ValueError(f"{name} must have unit innermost stride")
    return (T, heads, H), _lib.rows(t.data_ptr(), st, sk)


def _like(t: torch.Tensor) -> torch.Tensor:
    return torch.empty_strided(t.shape, t.stride(), dtype=t.dtype, device=t.device)


def _wdt(w: torch.Tensor) -> int:
    if w.dtype == torch.bfloat16:
        return _lib.RMS_BF16
    if w.dtype == torch.float32:
        return _lib.RMS_FP32
    raise TypeError(f"w must be bfloat16 or float32 (got {w.dtype})")


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def rmsnorm_train_fwd(x: torch.Tensor, w: torch.Tensor, eps: float = 1e-6,
                      residual: torch.Tensor | None = None, y: torch.Tensor | None = None,
                      rstd: torch.Tensor | None = None, h_out: torch.Tensor | None = None):
    """Forward.  Returns ``(y, rstd)``, or ``(h, y, rstd)`` with a residual."""
    (T, heads, H), xv = _view(x, "x")
    y = _like(x) if y is None else y
    _, yv = _view(y, "y")
    if rstd is None:
        rstd = torch.empty(T * heads, dtype=torch.float32, device=x.device)
    sh = _lib.shape(T, heads, H)
    L = _lib.lib()
    if residual is None:
        _lib.check(L.rms_train_fwd(sh, xv, w.data_ptr(), _wdt(w), yv, rstd.data_ptr(),
                                   float(eps), _stream()))
        return y, rstd
    _, rv = _view(residual, "residual")
    h_out = _like(x) if h_out is None else h_out
    _, hv = _view(h_out, "h_out")
    _lib.check(L.rms_residual_train_fwd(sh, xv, rv, w.data_ptr(), _wdt(w), hv, yv,
                                        rstd.data_ptr(), float(eps), _stream()))
    return h_out, y, rstd


class Workspace:
    """A zero-filled device buffer that grows on demand; reused across calls on one
    stream (the library leaves it ready for the next call)."""

    def __init__(self, device=None):
        self.device = torch.device(device if device is not None else "cuda")
        self.buf = torch.zeros(0, dtype=torch.uint8, device=self.device)

    def get(self, nbytes: int) -> torch.Tensor:
        if self.buf.numel() < nbytes:
            self.buf = torch.zeros(max(nbytes, 4096), dtype=torch.uint8, device=self.device)
        return self.buf


_default_ws: dict = {}


def _workspace_for(device) -> Workspace:
    key = torch.device(device)
    if key not in _default_ws:
        _default_ws[key] = Workspace(key)
    return _default_ws[key]


def rmsnorm_train_bwd(x: torch.Tensor, w: torch.Tensor, rstd: torch.Tensor, dy: torch.Tensor,
                      deterministic: bool = True, dh: torch.Tensor | None = None,
                      workspace: Workspace | None = None, grid_ctas: int = 0,
                      dx: torch.Tensor | None = None, dw: torch.Tensor | None = None):
    """Backward.  ``x`` is the forward input (h in the residual form).  Returns ``(dx, dw)``;
    with ``dh`` the first result is grad_h."""
    (T, heads, H), xv = _view(x, "x")
    _, dyv = _view(dy, "dy")
    dx = _like(x) if dx is None else dx
    _, dxv = _view(dx, "dx")
    if dw is None:
        dw = torch.empty(H, dtype=torch.float32, device=x.device)
    if rstd.dtype != torch.float32:
        raise TypeError("rstd must be float32")
    sh = _lib.shape(T, heads, H)
    L = _lib.lib()
    need = L.rms_train_bwd_workspace_bytes(sh, int(bool(deterministic)), int(grid_ctas))
    ws = (workspace or _workspace_for(x.device)).get(need)
    args = (w.data_ptr(), _wdt(w), rstd.data_ptr())
    if dh is None:
        rc = L.rms_train_bwd(sh, xv, *args, dyv, dxv, dw.data_ptr(), int(bool(deterministic)),
                             ws.data_ptr(), ws.numel(), int(grid_ctas), _stream())
    else:
        _, dhv = _view(dh, "dh")
        rc = L.rms_residual_train_bwd(sh, xv, *args, dyv, dhv, dxv, dw.data_ptr(),
                                      int(bool(deterministic)), ws.data_ptr(), ws.numel(),
                                      int(grid_ctas), _stream())
    _lib.check(rc)
    return dx, dw


def det_plan(T: int, heads: int, H: int):
    """(block_rows, blocks_per_chunk, fold_segments) of the deterministic order."""
    import ctypes
    b, l, s = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    _lib.check(_lib.lib().rms_det_plan(_lib.shape(T, heads, H), ctypes.byref(b),
                                       ctypes.byref(l), ctypes.byref(s)))
    return b.value, l.value, s.value


def bwd_path(T: int, heads: int, H: int, deterministic: bool) -> int:
    return int(_lib.lib().rms_train_bwd_path(_lib.shape(T, heads, H), int(bool(deterministic))))


def set_small_rows_limit(rows: int) -> int:
    return int(_lib.lib().rms_set_small_rows_limit(int(rows)))


def status(workspace: Workspace | None = None, device=None) -> None:
    """Raises RmsError if a backward on this workspace (the default one if None) recorded
    a device-side error; clears the word."""
    ws = workspace or _workspace_for(device if device is not None else "cuda")
    if ws.buf.numel() == 0:
        return
    _lib.check(_lib.lib().rms_status(ws.buf.data_ptr(), _stream()))


def forward_status() -> None:
    """Synchronises the current stream and raises RmsError on a CUDA error there (the
    forward kernels have no device-side waits and no status word of their own)."""
    _lib.check(_lib.lib().rms_status(None, _stream()))
