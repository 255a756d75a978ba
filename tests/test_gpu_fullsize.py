"""Full-size large-T workloads (the benchmark's shapes and launch configuration): the row
outputs are checked on sampled rows the oracle computes one by one, dw over every row,
and the deterministic bits across grids."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from bwd_rmsnorm_fwd_b200 import api, synth

from gpu_common import assert_dw, assert_dx, assert_fwd, dev_rows, dev_weight, host_bits

pytestmark = pytest.mark.gpu

EPS = 1e-6


def sample_idx(R, n=384, seed=0):
    g = np.random.default_rng(seed)
    idx = np.unique(np.concatenate([g.integers(0, R, n), [0, 1, R // 2, R - 2, R - 1]]))
    return idx[(idx >= 0) & (idx < R)]


@pytest.mark.parametrize("H,T,wdt", [(6144, 131072, "bf16"), (5120, 98304, "fp32"),
                                     (2048, 65537, "bf16")])
def test_large_t_full_size(H, T, wdt):
    x = synth.rows(11, "x", T, H)
    dy = synth.rows(11, "dy", T, H)
    w = synth.weight(11, H, wdt)
    idx = sample_idx(T)
    # oracle: forward on the sampled rows (rows are independent), rstd of every row for
    # the backward input, dw over every row
    y_ref_s, rstd_ref_s = oracle.train_fwd(x[idx], w)
    _, rstd_all = oracle.train_fwd(x, w)
    dx_ref_s, _ = oracle.train_bwd(x[idx], w, rstd_all[idx], dy[idx], want_dw=False)
    _, dw_ref = oracle.train_bwd(x, w, rstd_all, dy, want_dx=False)

    xd, dyd, wd = dev_rows(x), dev_rows(dy), dev_weight(w)
    del x, dy
    y, rstd = api.rmsnorm_train_fwd(xd, wd, EPS)
    torch.cuda.synchronize()
    it = torch.from_numpy(idx).cuda()
    assert_fwd(host_bits(y[it]), rstd[it].cpu().numpy(), y_ref_s, rstd_ref_s, "fwd sampled")
    del y
    rstd_in = torch.from_numpy(rstd_all).cuda()
    dws = {}
    for det in (False, True):
        dx, dw = api.rmsnorm_train_bwd(xd, wd, rstd_in, dyd, deterministic=det)
        api.status()
        torch.cuda.synchronize()
        assert_dx(host_bits(dx[it]), dx_ref_s, f"dx sampled det={det}")
        assert_dw(dw.cpu().numpy(), dw_ref, f"dw det={det}")
        dws[det] = dw.cpu().numpy()
        del dx
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for grid in (sms // 2, sms + 3, 4 * sms):
        _, dw = api.rmsnorm_train_bwd(xd, wd, rstd_in, dyd, deterministic=True, grid_ctas=grid)
        assert np.array_equal(dw.cpu().numpy().view(np.uint32), dws[True].view(np.uint32)), grid
