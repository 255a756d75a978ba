"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module only draws random numbers and lays them out; it holds none of the
RMSNorm arithmetic.  Inputs are generated in blocks of ``BLOCK_ROWS`` rows, each
block from its own counter-based seed ``(seed, tensor name, block index)``, so a
checker can regenerate any subset of rows of a large tensor without drawing the
rest.

Input families (the pages' dw sweeps run "three input families" without defining
them; these are the readings used here):

* ``F1`` -- x, dy, residual, dh ~ N(0, 1), cast to BF16 (nearest-even).
* ``F2`` -- heavy-tailed: F1, then 1 % of the x entries are scaled by 64 and the dy
  rows of 1 % of the rows are scaled by 16.
* ``F3`` -- cancellation-heavy: rows come in pairs with equal x and
  ``dy[2i+1] = -dy[2i] * (1 + 2^-8 N(0,1))``, so every dw column nearly cancels.

The weight is ``1 + 0.1 N(0,1)`` drawn in FP32 and, for a BF16 weight, cast to BF16.
"""

from __future__ import annotations

import zlib

import numpy as np
import torch

BLOCK_ROWS = 1024  # even, so F3 row pairs never straddle a block

_NAMES = {"x": 1, "dy": 2, "res": 3, "dh": 4, "w": 5}


def _rng(seed: int, name: str, block: int) -> np.random.Generator:
    tag = _NAMES.get(name) or (zlib.crc32(name.encode()) & 0x7FFFFFFF)
    return np.random.default_rng(np.random.SeedSequence([int(seed), int(tag), int(block)]))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """FP32 -> BF16 bits (nearest-even) through torch's conversion."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _block(seed: int, name: str, block: int, H: int, family: str) -> np.ndarray:
    """FP32 values of rows [block*BLOCK_ROWS, (block+1)*BLOCK_ROWS) of tensor ``name``."""
    g = _rng(seed, name, block)
    v = g.standard_normal((BLOCK_ROWS, H), dtype=np.float32)
    if family == "F1":
        return v
    if family == "F2":
        if name == "x":
            mask = g.random((BLOCK_ROWS, H)) < 0.01
            v[mask] *= 64.0
        elif name == "dy":
            rows = g.random(BLOCK_ROWS) < 0.01
            v[rows] *= 16.0
        return v
    if family == "F3":
        if name == "x":
            v[1::2] = v[0::2]
        elif name == "dy":
            jitter = g.standard_normal((BLOCK_ROWS // 2, H), dtype=np.float32)
            v[1::2] = -v[0::2] * (np.float32(1.0) + np.float32(2.0 ** -8) * jitter)
        return v
    raise ValueError(f"unknown input family {family!r}")


def rows(seed: int, name: str, R: int, H: int, family: str = "F1", row0: int = 0,
         nrows: int | None = None) -> np.ndarray:
    """BF16 bits ``[nrows, H]`` of rows ``row0 ...`` of the conceptual ``[R, H]`` tensor."""
    if nrows is None:
        nrows = R - row0
    assert 0 <= row0 and row0 + nrows <= R
    out = np.empty((nrows, H), np.uint16)
    r = row0
    while r < row0 + nrows:
        b = r // BLOCK_ROWS
        b0 = b * BLOCK_ROWS
        take = min(row0 + nrows, b0 + BLOCK_ROWS) - r
        blk = f32_to_bf16_bits(_block(seed, name, b, H, family)[r - b0: r - b0 + take])
        out[r - row0: r - row0 + take] = blk
        r += take
    return out


def sample_rows(seed: int, name: str, R: int, H: int, idx, family: str = "F1") -> np.ndarray:
    """BF16 bits of the rows listed in ``idx`` (any order), regenerating only their blocks."""
    idx = np.asarray(idx, dtype=np.int64)
    out = np.empty((idx.size, H), np.uint16)
    cache: dict[int, np.ndarray] = {}
    for i, r in enumerate(idx.tolist()):
        b = r // BLOCK_ROWS
        if b not in cache:
            cache[b] = f32_to_bf16_bits(_block(seed, name, b, H, family))
        out[i] = cache[b][r - b * BLOCK_ROWS]
    return out


def weight(seed: int, H: int, dtype: str) -> np.ndarray:
    """``1 + 0.1 N(0,1)``: uint16 BF16 bits for ``dtype='bf16'``, float32 for ``'fp32'``."""
    g = _rng(seed, "w", 0)
    w = (np.float32(1.0) + np.float32(0.1) * g.standard_normal(H, dtype=np.float32))
    if dtype == "bf16":
        return f32_to_bf16_bits(w)
    if dtype == "fp32":
        return w.astype(np.float32)
    raise ValueError(dtype)


# ---- layouts --------------------------------------------------------------------------

def view_extent(T: int, heads: int, H: int, st: int, sk: int) -> int:
    """Elements spanned by a ``[T, heads, H]`` view with strides ``(st, sk, 1)``."""
    if T == 0:
        return 0
    return (T - 1) * st + (heads - 1) * sk + H


def place_rows(rows_u16: np.ndarray, T: int, heads: int, H: int, st: int, sk: int,
               fill: int = 0x7FC1) -> np.ndarray:
    """Scatter dense rows ``[T*heads, H]`` into a flat BF16-bit buffer laid out with
    strides ``(st, sk, 1)``; elements outside the view hold ``fill`` (a NaN pattern)."""
    n = view_extent(T, heads, H, st, sk)
    buf = np.full(max(n, 1), fill, np.uint16)
    if T:
        idx = (np.arange(T)[:, None] * st + np.arange(heads)[None, :] * sk).reshape(-1)
        buf[idx[:, None] + np.arange(H)[None, :]] = rows_u16
    return buf


def gather_rows(buf_u16: np.ndarray, T: int, heads: int, H: int, st: int, sk: int) -> np.ndarray:
    """Inverse of :func:`place_rows`: dense ``[T*heads, H]`` rows out of a flat buffer."""
    if T == 0:
        return np.empty((0, H), np.uint16)
    idx = (np.arange(T)[:, None] * st + np.arange(heads)[None, :] * sk).reshape(-1)
    return buf_u16[idx[:, None] + np.arange(H)[None, :]]
