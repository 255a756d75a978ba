"""Shared helpers for the GPU tests: device tensors from seeded BF16 bits, oracle runs,
and the comparison rules.

Tolerances (flashinfer PR #8848 "Measurement": dx atol = rtol = 1e-2, dw per element
atol 1e-4 + rtol 1e-4 against FP64), plus, for outputs the pages fix only by dtype:
y within one BF16 ulp of the oracle's correctly rounded value (the GPU rounds an FP32
product whose error is ~3e-7 relative, so it can land on the other side of a rounding
boundary but never further), rstd within 2e-6 relative (FP32 sum of exact squares: a
summation depth <= 40 gives <= 40 * 2^-24 relative on the mean, half of that on rstd,
plus one rounding of the scaled mean and rsqrtf's documented 2 ulp), h bit-exact (the
sum of two BF16 values is exact in FP32 whenever it can matter, so one rounding gives the oracle's bits).
"""

from __future__ import annotations

import numpy as np
import torch

import oracle
from bwd_rmsnorm_fwd_b200 import synth

DX_ATOL = DX_RTOL = 1e-2
DW_ATOL = DW_RTOL = 1e-4
RSTD_RTOL = 2e-6

DEV = "cuda"


def dev_rows(bits: np.ndarray) -> torch.Tensor:
    """Dense [R, H] BF16 device tensor from BF16 bits."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(DEV)


def dev_weight(w: np.ndarray) -> torch.Tensor:
    if w.dtype == np.uint16:
        return torch.from_numpy(w.view(np.int16)).view(torch.bfloat16).to(DEV)
    return torch.from_numpy(w).to(DEV)


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def strided_buffer(rows_bits: np.ndarray, T: int, heads: int, H: int, st: int, sk: int,
                   fill: int = 0x7FC1):
    """A poison-filled device buffer holding the rows at strides (st, sk, 1), and the
    [T, heads, H] view into it."""
    flat = synth.place_rows(rows_bits, T, heads, H, st, sk, fill)
    buf = dev_rows(flat.reshape(1, -1)).reshape(-1)
    view = torch.as_strided(buf, (T, heads, H), (st, sk, 1))
    return buf, view


def empty_strided_buffer(T: int, heads: int, H: int, st: int, sk: int, fill: int = 0x7FC1):
    n = max(synth.view_extent(T, heads, H, st, sk), 1)
    buf = torch.full((n,), 0, dtype=torch.int16, device=DEV)
    buf.fill_(np.int16(np.uint16(fill).view(np.int16)).item())
    buf = buf.view(torch.bfloat16)
    view = torch.as_strided(buf, (T, heads, H), (st, sk, 1))
    return buf, view


def view_rows(view: torch.Tensor) -> np.ndarray:
    """Dense [R, H] bits of a [T, heads, H] (or [T, H]) device view."""
    H = view.shape[-1]
    return host_bits(view.reshape(-1, H) if view.is_contiguous() else view.contiguous().reshape(-1, H))


def gaps_untouched(buf: torch.Tensor, T: int, heads: int, H: int, st: int, sk: int,
                   fill: int = 0x7FC1) -> bool:
    """True when every element of buf outside the view still holds the fill pattern."""
    b = host_bits(buf)
    mask = np.ones(b.size, bool)
    if T:
        idx = (np.arange(T)[:, None] * st + np.arange(heads)[None, :] * sk).reshape(-1)
        mask[(idx[:, None] + np.arange(H)[None, :]).reshape(-1)] = False
    return bool(np.all(b[mask] == fill))


def ordered(bits: np.ndarray) -> np.ndarray:
    b = bits.astype(np.int32)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


def bf16_ulps(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    return np.abs(ordered(a) - ordered(b))


def f32(bits: np.ndarray) -> np.ndarray:
    return synth.bf16_bits_to_f32(bits)


def assert_fwd(y_bits, rstd, y_ref, rstd_ref, what=""):
    u = bf16_ulps(y_bits, y_ref)
    assert u.max(initial=0) <= 1, f"{what}: y differs by {u.max()} BF16 ulps"
    rel = np.abs(rstd.astype(np.float64) - rstd_ref) / np.abs(rstd_ref)
    assert rel.max(initial=0) <= RSTD_RTOL, f"{what}: rstd rel err {rel.max():.3g}"


def assert_dx(dx_bits, dx_ref_bits, what=""):
    a, b = f32(dx_bits).astype(np.float64), f32(dx_ref_bits).astype(np.float64)
    err = np.abs(a - b)
    tol = DX_ATOL + DX_RTOL * np.abs(b)
    assert np.all(err <= tol), f"{what}: dx worst err/tol {np.max(err / tol):.3g}"
    # a systematic error shows in the mean long before it reaches the budget
    if b.size:
        assert err.mean() <= 2e-3 * max(np.abs(b).mean(), 1e-30), f"{what}: dx mean error"


def dw_ratio(dw: np.ndarray, dw_ref64: np.ndarray) -> float:
    """Worst per-element |err| / (atol + rtol |ref|) against the FP64 oracle."""
    err = np.abs(dw.astype(np.float64) - dw_ref64)
    return float(np.max(err / (DW_ATOL + DW_RTOL * np.abs(dw_ref64)), initial=0.0))


def assert_dw(dw, dw_ref64, what=""):
    r = dw_ratio(dw, dw_ref64)
    assert r <= 1.0, f"{what}: dw worst err/tol {r:.3g}"
