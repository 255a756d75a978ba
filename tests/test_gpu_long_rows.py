"""The very long narrow-row regime: H 256 rows at T 1,048,576 (the pages' H256 T1048576 rows,
BF16 and FP32 weight), both backward modes.  Row outputs are checked on sampled rows the
oracle computes one by one, dw over every row; the deterministic bits across three grids
(the order's 64-row blocks in 2048 chunks at this size); and the blocked-FP32 program's
cut-over at 2^24 elements from both sides, against the full oracle."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from bwd_rmsnorm_fwd_b200 import api, synth

from gpu_common import assert_dw, assert_dx, assert_fwd, dev_rows, dev_weight, host_bits

pytestmark = pytest.mark.gpu


def sample_idx(R, n=512, seed=1):
    g = np.random.default_rng(seed)
    idx = np.unique(np.concatenate([g.integers(0, R, n), [0, 1, 63, 64, R // 2, R - 2, R - 1]]))
    return idx[(idx >= 0) & (idx < R)]


@pytest.mark.parametrize("wdt", ["bf16", "fp32"])
def test_h256_million_rows(wdt):
    T, H = 1 << 20, 256
    B, L, S = api.det_plan(T, 1, H)
    assert (B, L, S) == (64, 8, 16)             # 2048 chunks of 512 rows
    x = synth.rows(80, "x", T, H)
    dy = synth.rows(80, "dy", T, H)
    w = synth.weight(80, H, wdt)
    idx = sample_idx(T)
    y_ref_s, rstd_ref_s = oracle.train_fwd(x[idx], w)
    _, rstd_all = oracle.train_fwd(x, w)
    dx_ref_s, _ = oracle.train_bwd(x[idx], w, rstd_all[idx], dy[idx], want_dw=False)
    _, dw_ref = oracle.train_bwd(x, w, rstd_all, dy, want_dx=False)
    xd, dyd, wd = dev_rows(x), dev_rows(dy), dev_weight(w)
    del x, dy
    y, rstd = api.rmsnorm_train_fwd(xd, wd)
    torch.cuda.synchronize()
    it = torch.from_numpy(idx).cuda()
    assert_fwd(host_bits(y[it]), rstd[it].cpu().numpy(), y_ref_s, rstd_ref_s, "fwd sampled")
    del y
    rs = torch.from_numpy(rstd_all).cuda()
    dws = {}
    for det in (True, False):
        assert api.bwd_path(T, 1, H, det) == (2 if det else 3)
        dx, dw = api.rmsnorm_train_bwd(xd, wd, rs, dyd, deterministic=det)
        api.status()
        assert_dx(host_bits(dx[it]), dx_ref_s, f"dx sampled det={det}")
        assert_dw(dw.cpu().numpy(), dw_ref, f"dw det={det}")
        dws[det] = dw.cpu().numpy()
        del dx
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for grid in (sms // 2, sms + 5, 1000):
        _, dw = api.rmsnorm_train_bwd(xd, wd, rs, dyd, deterministic=True, grid_ctas=grid)
        assert np.array_equal(dw.cpu().numpy().view(np.uint32), dws[True].view(np.uint32)), grid


@pytest.mark.parametrize("T", [65535, 65536, 65537])
def test_blocked_fp32_cut_over_at_2_24_elements(T):
    """H 256 just below, at and above 2^24 elements: the one-warp-per-row program below, the
    bulk-copy pipeline from there on; both against the full oracle."""
    H = 256
    x = synth.rows(81, "x", T, H)
    dy = synth.rows(81, "dy", T, H)
    w = synth.weight(81, H, "bf16")
    _, rstd = oracle.train_fwd(x, w)
    dx_ref, dw_ref = oracle.train_bwd(x, w, rstd, dy)
    dx, dw = api.rmsnorm_train_bwd(dev_rows(x), dev_weight(w), torch.from_numpy(rstd).cuda(),
                                   dev_rows(dy), deterministic=False)
    api.status()
    assert_dx(host_bits(dx), dx_ref, f"dx T={T}")
    assert_dw(dw.cpu().numpy(), dw_ref, f"dw T={T}")
