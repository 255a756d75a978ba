"""Deterministic dw: bit-identical across grids, repeats and programs, and equal bit for
bit to a CPU emulation of the documented summation order (a test of the order, kept
apart from the FP64 oracle, which defines the value)."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from bwd_rmsnorm_fwd_b200 import api, synth

from det_order import emulate_det_dw
from gpu_common import dev_rows, dev_weight

pytestmark = pytest.mark.gpu


def inputs(T, heads, H, seed=0, family="F1", wdt="bf16"):
    R = T * heads
    x = synth.rows(seed, "x", R, H, family)
    dy = synth.rows(seed, "dy", R, H, family)
    w = synth.weight(seed, H, wdt)
    _, rstd = oracle.train_fwd(x, w)
    return x, dy, w, rstd


def gpu_dw(x, dy, w, rstd, det=True, grid=0, heads=1, res_dh=None):
    H = x.shape[1]
    xd = dev_rows(x).reshape(-1, heads, H) if heads > 1 else dev_rows(x)
    dyd = dev_rows(dy).reshape(xd.shape)
    dh = None if res_dh is None else dev_rows(res_dh).reshape(xd.shape)
    _, dw = api.rmsnorm_train_bwd(xd, dev_weight(w), torch.from_numpy(rstd).cuda(), dyd,
                                  deterministic=det, grid_ctas=grid, dh=dh)
    torch.cuda.synchronize()
    return dw.cpu().numpy()


@pytest.mark.parametrize("T,heads,H", [(70001, 1, 6144), (9000, 1, 1536), (4096, 24, 256),
                                       (20000, 1, 4096), (50000, 1, 2048), (30000, 4, 256)])
def test_bits_identical_across_grids_and_repeats(T, heads, H):
    x, dy, w, rstd = inputs(T, heads, H, seed=5, family="F3")
    ref = gpu_dw(x, dy, w, rstd, heads=heads)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for grid in (1, 7, 37, sms, 2 * sms, 3 * sms + 1, 1000):
        got = gpu_dw(x, dy, w, rstd, grid=grid, heads=heads)
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32)), grid
    for _ in range(3):
        assert np.array_equal(gpu_dw(x, dy, w, rstd, heads=heads).view(np.uint32),
                              ref.view(np.uint32))


@pytest.mark.parametrize("T,H", [(227, 4096), (1000, 512), (2048, 256), (600, 1536)])
def test_single_launch_and_pair_give_the_same_bits(T, H):
    x, dy, w, rstd = inputs(T, 1, H, seed=6, family="F2")
    prev = api.set_small_rows_limit(1 << 30)
    try:
        assert api.bwd_path(T, 1, H, True) == 1
        a = gpu_dw(x, dy, w, rstd)
        api.set_small_rows_limit(0)
        assert api.bwd_path(T, 1, H, True) == 2
        b = gpu_dw(x, dy, w, rstd)
        c = gpu_dw(x, dy, w, rstd, grid=3)
    finally:
        api.set_small_rows_limit(prev)
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    assert np.array_equal(a.view(np.uint32), c.view(np.uint32))


@pytest.mark.parametrize("T,heads,H", [(227, 1, 512), (5000, 1, 1536), (4100, 1, 6144),
                                       (700, 24, 256), (33000, 1, 264), (6000, 1, 2048),
                                       (2500, 1, 4096), (3000, 1, 5120), (2000, 1, 8192)])
def test_bits_equal_cpu_emulation_of_the_order(T, heads, H):
    x, dy, w, rstd = inputs(T, heads, H, seed=7, family="F3", wdt="fp32")
    B, L, S = api.det_plan(T, heads, H)
    want = emulate_det_dw(x, dy, rstd, B, L, S)
    got = gpu_dw(x, dy, w, rstd, heads=heads)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def test_residual_form_bits_do_not_depend_on_grid():
    T, H = 5000, 6144
    x, dy, w, rstd = inputs(T, 1, H, seed=8)
    dh = synth.rows(8, "dh", T, H)
    ref = gpu_dw(x, dy, w, rstd, res_dh=dh)
    for grid in (5, 148, 999):
        assert np.array_equal(gpu_dw(x, dy, w, rstd, grid=grid, res_dh=dh).view(np.uint32),
                              ref.view(np.uint32))
