"""An IEEE emulation of the deterministic dw order (a test of the order, kept apart from the
FP64 oracle, which defines the value): numpy FP32 and FP64 operations only, each rounding to
nearest like the kernels' explicit-rounding intrinsics."""

from __future__ import annotations

import numpy as np

from bwd_rmsnorm_fwd_b200 import synth


def emulate_det_dw(x_bits, dy_bits, rstd, B, L, S):
    """IEEE emulation of the fixed order: per column, blocks of B rows summed in row order
    with exact products (p + e == dy * xh) and TwoSum; each block -> FP64 (s + c); L blocks
    per chunk folded left to right; S contiguous segments of chunks folded left to right;
    the segment sums folded left to right; one rounding to FP32."""
    x = synth.bf16_bits_to_f32(x_bits)
    dy = synth.bf16_bits_to_f32(dy_bits)
    R, H = x.shape
    rstd = rstd.astype(np.float32)
    n_blocks = -(-R // B)
    bp = np.empty((n_blocks, H), np.float64)
    for b in range(n_blocks):
        s = np.zeros(H, np.float32)
        c = np.zeros(H, np.float32)
        for r in range(b * B, min(R, (b + 1) * B)):
            xh = x[r] * rstd[r]                                   # FP32, nearest
            p = dy[r] * xh
            e = (dy[r].astype(np.float64) * xh.astype(np.float64) - p).astype(np.float32)
            t = s + p
            z = t - s
            err = (s - (t - z)) + (p - z)
            c = c + (err + e)
            s = t
        bp[b] = s.astype(np.float64) + c.astype(np.float64)
    n_chunks = -(-n_blocks // L)
    chunks = []
    for k in range(n_chunks):
        a = bp[k * L].copy()
        for b in range(k * L + 1, min(n_blocks, (k + 1) * L)):
            a = a + bp[b]
        chunks.append(a)
    seg_len = -(-n_chunks // S)
    total = None
    for q in range(S):
        k0, k1 = q * seg_len, min(n_chunks, (q + 1) * seg_len)
        if k0 >= k1:
            continue
        sg = chunks[k0].copy()
        for k in range(k0 + 1, k1):
            sg = sg + chunks[k]
        total = sg if total is None else total + sg
    return total.astype(np.float32)


def emulate_chunk_partials(x_bits, dy_bits, rstd, B, L):
    """FP64 chunk partials [n_chunks, H] of the fixed order over the given rows (blocks of B
    rows summed with exact products and TwoSum, L blocks per chunk folded left to right)."""
    x = synth.bf16_bits_to_f32(x_bits)
    dy = synth.bf16_bits_to_f32(dy_bits)
    R, H = x.shape
    rstd = rstd.astype(np.float32)
    n_blocks = -(-R // B)
    bp = np.empty((n_blocks, H), np.float64)
    for b in range(n_blocks):
        s = np.zeros(H, np.float32)
        c = np.zeros(H, np.float32)
        for r in range(b * B, min(R, (b + 1) * B)):
            xh = x[r] * rstd[r]
            p = dy[r] * xh
            e = (dy[r].astype(np.float64) * xh.astype(np.float64) - p).astype(np.float32)
            t = s + p
            z = t - s
            err = (s - (t - z)) + (p - z)
            c = c + (err + e)
            s = t
        bp[b] = s.astype(np.float64) + c.astype(np.float64)
    n_chunks = -(-n_blocks // L)
    out = np.empty((n_chunks, H), np.float64)
    for k in range(n_chunks):
        a = bp[k * L].copy()
        for b in range(k * L + 1, min(n_blocks, (k + 1) * L)):
            a = a + bp[b]
        out[k] = a
    return out


def emulate_segment_sums(chunks, seg_len, n_seg):
    """Sums of n_seg consecutive segments of seg_len chunk partials each (left to right), the
    segments starting at the first chunk given; 0 for a segment with no chunks."""
    H = chunks.shape[1]
    out = np.zeros((n_seg, H), np.float64)
    for q in range(n_seg):
        k0, k1 = q * seg_len, min(len(chunks), (q + 1) * seg_len)
        if k0 >= k1:
            continue
        a = chunks[k0].copy()
        for k in range(k0 + 1, k1):
            a = a + chunks[k]
        out[q] = a
    return out


def emulate_fold_table(table, n_nonempty):
    """The final fold: the first n_nonempty segment sums left to right, one FP32 rounding."""
    tot = table[0].copy()
    for q in range(1, n_nonempty):
        tot = tot + table[q]
    return tot.astype(np.float32)
