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
    "rmsnorm_train_fwd", "rmsnorm_train_bwd", "rmsnorm_train", "RMSNormTrainFunction",
    "Workspace", "det_plan", "bwd_path", "set_small_rows_limit", "status", "forward_status",
    "record_backward_events", "shard_rows", "gather_segments", "rmsnorm_train_bwd_det_shard",
    "fold_segments", "rmsnorm_train_bwd_sharded",
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
                      dx: torch.Tensor | None = None, dw: torch.Tensor | None = None,
                      accumulate: bool = False):
    """Backward.  ``x`` is the forward input (h in the residual form).  Returns ``(dx, dw)``;
    with ``dh`` the first result is grad_h.  With ``accumulate`` the call adds into the given
    FP32 ``dw``: dw = FP32(dw + the dw the overwrite call returns)."""
    (T, heads, H), xv = _view(x, "x")
    _, dyv = _view(dy, "dy")
    dx = _like(x) if dx is None else dx
    _, dxv = _view(dx, "dx")
    if dw is None:
        if accumulate:
            raise ValueError("accumulate=True needs the dw buffer to add into")
        dw = torch.empty(H, dtype=torch.float32, device=x.device)
    if dw.dtype != torch.float32 or dw.numel() != H or not dw.is_contiguous():
        raise ValueError("dw must be a contiguous float32 tensor of H elements")
    if rstd.dtype != torch.float32:
        raise TypeError("rstd must be float32")
    sh = _lib.shape(T, heads, H)
    L = _lib.lib()
    need = L.rms_train_bwd_workspace_bytes(sh, int(bool(deterministic)), int(grid_ctas))
    ws = (workspace or _workspace_for(x.device)).get(need)
    args = (w.data_ptr(), _wdt(w), rstd.data_ptr())
    if dh is None:
        f = L.rms_train_bwd_accumulate if accumulate else L.rms_train_bwd
        rc = f(sh, xv, *args, dyv, dxv, dw.data_ptr(), int(bool(deterministic)),
               ws.data_ptr(), ws.numel(), int(grid_ctas), _stream())
    else:
        _, dhv = _view(dh, "dh")
        f = L.rms_residual_train_bwd_accumulate if accumulate else L.rms_residual_train_bwd
        rc = f(sh, xv, *args, dyv, dhv, dxv, dw.data_ptr(), int(bool(deterministic)),
               ws.data_ptr(), ws.numel(), int(grid_ctas), _stream())
    _lib.check(rc)
    return dx, dw


# ---- row sharding over ranks, deterministic ------------------------------------------------

FOLD_SEGMENTS = 16


def shard_rows(T: int, H: int, rank: int, world: int):
    """(row_begin, row_end, workspace_bytes) of `rank` in a row-sharded deterministic backward
    of T rows of width H over `world` ranks (world divides 16)."""
    import ctypes
    b, e, ws = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_size_t()
    _lib.check(_lib.lib().rms_det_shard_plan(_lib.shape(T, 1, H), int(rank), int(world),
                                             ctypes.byref(b), ctypes.byref(e), ctypes.byref(ws)))
    return b.value, e.value, ws.value


def gather_segments(seg_local: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather of every rank's segment sums, in rank order (= segment order): the
    [16, H] FP64 table.  NCCL's all_gather_into_tensor for device tensors, gloo's all_gather
    for host tensors."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    out = torch.empty((world * seg_local.shape[0], seg_local.shape[1]), dtype=seg_local.dtype,
                      device=seg_local.device)
    if seg_local.is_cuda:
        dist.all_gather_into_tensor(out, seg_local.contiguous(), group=group)
    else:
        dist.all_gather(list(out.chunk(world)), seg_local.contiguous(), group=group)
    return out


def rmsnorm_train_bwd_det_shard(x: torch.Tensor, w: torch.Tensor, rstd: torch.Tensor,
                                dy: torch.Tensor, T: int, rank: int, world: int,
                                dh: torch.Tensor | None = None,
                                workspace: Workspace | None = None, grid_ctas: int = 0,
                                dx: torch.Tensor | None = None):
    """This rank's part of a row-sharded deterministic backward of T rows: x, dy (dh) and
    rstd hold the rank's rows (shard_rows).  Returns (dx, seg) with seg the rank's FP64
    segment sums [16 // world, H]."""
    (Tl, heads, H), xv = _view(x, "x")
    if heads != 1:
        raise ValueError("row sharding takes [T, H] rows")
    b, e, need = shard_rows(T, H, rank, world)
    if Tl != e - b:
        raise ValueError(f"rank {rank} owns rows [{b}, {e}): got {Tl} rows")
    _, dyv = _view(dy, "dy")
    dx = _like(x) if dx is None else dx
    _, dxv = _view(dx, "dx")
    dhv = _view(dh, "dh")[1] if dh is not None else _lib.rows(0, 0, 0)
    seg = torch.empty((FOLD_SEGMENTS // world, H), dtype=torch.float64, device=x.device)
    ws = (workspace or _workspace_for(x.device)).get(need)
    _lib.check(_lib.lib().rms_train_bwd_det_shard(
        _lib.shape(T, 1, H), int(rank), int(world), xv, w.data_ptr(), _wdt(w), rstd.data_ptr(),
        dyv, dhv, dxv, seg.data_ptr(), ws.data_ptr(), ws.numel(), int(grid_ctas), _stream()))
    return dx, seg


def fold_segments(seg: torch.Tensor, T: int, H: int, dw: torch.Tensor | None = None,
                  accumulate: bool = False) -> torch.Tensor:
    """dw of the whole T-row problem from the [16, H] table of segment sums."""
    if seg.dtype != torch.float64 or tuple(seg.shape) != (FOLD_SEGMENTS, H) or not seg.is_contiguous():
        raise ValueError("seg must be a contiguous float64 [16, H] table")
    if dw is None:
        if accumulate:
            raise ValueError("accumulate=True needs the dw buffer to add into")
        dw = torch.empty(H, dtype=torch.float32, device=seg.device)
    _lib.check(_lib.lib().rms_det_fold_segments(_lib.shape(T, 1, H), seg.data_ptr(),
                                                dw.data_ptr(), int(bool(accumulate)), _stream()))
    return dw


def rmsnorm_train_bwd_sharded(x: torch.Tensor, w: torch.Tensor, rstd: torch.Tensor,
                              dy: torch.Tensor, T: int, dh: torch.Tensor | None = None,
                              group=None, workspace: Workspace | None = None,
                              dw: torch.Tensor | None = None, accumulate: bool = False):
    """Deterministic backward of T rows sharded over the ranks of `group` (torch.distributed):
    this rank passes its rows (shard_rows), gets its dx and the dw of all T rows, bit-identical
    to the single-GPU deterministic backward.  One collective: the all-gather of the FP64
    segment sums (16 x H x 8 bytes in all)."""
    import torch.distributed as dist
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    dx, seg = rmsnorm_train_bwd_det_shard(x, w, rstd, dy, T, rank, world, dh=dh,
                                          workspace=workspace)
    table = gather_segments(seg, group)
    return dx, fold_segments(table, T, x.shape[-1], dw=dw, accumulate=accumulate)


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


# ---- autograd -----------------------------------------------------------------------------

_bwd_event_log: list | None = None


class record_backward_events:
    """Context manager: while active, every backward run by :class:`RMSNormTrainFunction`
    records a pair of CUDA timing events on its stream around its library call and appends
    ``(start, end)`` to the given list (how long the backward kernels took inside a step
    driven by autograd)."""

    def __init__(self, log: list):
        self.log = log

    def __enter__(self):
        global _bwd_event_log
        self.prev, _bwd_event_log = _bwd_event_log, self.log
        return self.log

    def __exit__(self, *exc):
        global _bwd_event_log
        _bwd_event_log = self.prev
        return False


class RMSNormTrainFunction(torch.autograd.Function):
    """Training RMSNorm as an autograd function over the C ABI: the forward is
    rms_train_fwd (or rms_residual_train_fwd), the backward rms_train_bwd (or the residual
    backward).  Saves x (h), w and the FP32 rstd; under activation checkpointing the forward
    is simply run again.  With ``main_grad`` (a float32 [H] buffer) the backward adds dw into
    it with the accumulate entry point and gives w no gradient; otherwise w's gradient is
    the FP32 dw (autograd casts it to w's dtype)."""

    @staticmethod
    def forward(ctx, x, w, residual, eps, deterministic, main_grad, workspace):
        if residual is None:
            y, rstd = rmsnorm_train_fwd(x, w, eps)
            h = x
            outs = (y,)
        else:
            h, y, rstd = rmsnorm_train_fwd(x, w, eps, residual=residual)
            outs = (y, h)
        ctx.save_for_backward(h, w, rstd)
        ctx.residual = residual is not None
        ctx.deterministic = bool(deterministic)
        ctx.main_grad = main_grad
        ctx.workspace = workspace
        return outs if ctx.residual else y

    @staticmethod
    def backward(ctx, dy, dh=None):
        h, w, rstd = ctx.saved_tensors
        dy = dy.contiguous() if dy.stride(-1) != 1 else dy
        if ctx.residual:
            dh = torch.zeros_like(h) if dh is None else dh
            dh = dh.contiguous() if dh.stride(-1) != 1 else dh
        log = _bwd_event_log
        if log is not None:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
        acc = ctx.main_grad is not None
        dx, dw = rmsnorm_train_bwd(h, w, rstd, dy, deterministic=ctx.deterministic,
                                   dh=dh if ctx.residual else None,
                                   workspace=ctx.workspace, dw=ctx.main_grad if acc else None,
                                   accumulate=acc)
        if log is not None:
            b.record()
            log.append((a, b))
        gw = None if acc else dw
        if ctx.residual:
            return dx, gw, dx, None, None, None, None
        return dx, gw, None, None, None, None, None


def rmsnorm_train(x: torch.Tensor, w: torch.Tensor, eps: float = 1e-6,
                  residual: torch.Tensor | None = None, deterministic: bool = True,
                  main_grad: torch.Tensor | None = None, workspace: Workspace | None = None):
    """Differentiable training RMSNorm.  Returns y, or ``(y, h)`` with a residual (h = x +
    residual rounded to BF16; the gradient of h flows back to both x and residual)."""
    if main_grad is not None and (main_grad.dtype != torch.float32 or
                                  main_grad.numel() != w.numel()):
        raise ValueError("main_grad must be a float32 tensor with one element per column")
    return RMSNormTrainFunction.apply(x, w, residual, eps, deterministic, main_grad, workspace)
