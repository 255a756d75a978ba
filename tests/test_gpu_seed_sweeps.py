"""dw against the FP64 oracle over many seeds: the budget is a worst case over seeds
(flashinfer PR #8848 "Measurement": per element atol 1e-4 + rtol 1e-4, worst of the
seeds), so a single lucky seed proves little.

* small-T single-launch program, deterministic mode: 120 seeds at H 512 and H 4096;
* large T, both backward programs, the three input families (F1 Gaussian, F2 heavy-tailed,
  F3 cancellation-heavy): deterministic dw must meet the budget on every family; the
  blocked-FP32 mode must meet it on F1, and its F2/F3 ratios are reported (the pages hold
  the blocked mode to the budget on ordinary inputs only)."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from bwd_rmsnorm_fwd_b200 import api, synth

from gpu_common import dev_rows, dev_weight, dw_ratio

pytestmark = pytest.mark.gpu


def dw_runs(x, dy, w, modes, ws):
    """The oracle's FP64 dw and the GPU dw of each mode (oracle rstd in, as in every parity
    test)."""
    _, rstd = oracle.train_fwd(x, w)
    _, ref = oracle.train_bwd(x, w, rstd, dy, want_dx=False)
    xd, dyd, wd, rs = dev_rows(x), dev_rows(dy), dev_weight(w), torch.from_numpy(rstd).cuda()
    out = {}
    for det in modes:
        _, dw = api.rmsnorm_train_bwd(xd, wd, rs, dyd, deterministic=det, workspace=ws)
        api.status(ws)
        out[det] = dw.cpu().numpy()
    return ref, out


@pytest.mark.parametrize("H,T", [(512, 32), (512, 227), (4096, 32), (4096, 227)])
def test_small_t_dw_over_120_seeds(H, T):
    assert api.bwd_path(T, 1, H, True) == 1  # the single-launch program
    ws = api.Workspace("cuda")
    worst = 0.0
    for seed in range(120):
        x = synth.rows(1000 + seed, "x", T, H)
        dy = synth.rows(1000 + seed, "dy", T, H)
        w = synth.weight(1000 + seed, H, "bf16" if seed % 2 else "fp32")
        ref, dw = dw_runs(x, dy, w, (True,), ws)
        worst = max(worst, dw_ratio(dw[True], ref))
    print(f"H{H} T{T}: worst dw err/tol over 120 seeds {worst:.3g}")
    assert worst <= 1.0


@pytest.mark.parametrize("H,T", [(1536, 65537), (6144, 32768)])
def test_large_t_dw_families_over_seeds(H, T):
    ws = api.Workspace("cuda")
    report = {}
    for family in ("F1", "F2", "F3"):
        worst = {True: 0.0, False: 0.0}
        for seed in range(3):
            x = synth.rows(2000 + seed, "x", T, H, family)
            dy = synth.rows(2000 + seed, "dy", T, H, family)
            w = synth.weight(2000 + seed, H, "bf16")
            ref, dw = dw_runs(x, dy, w, (True, False), ws)
            for det in (True, False):
                worst[det] = max(worst[det], dw_ratio(dw[det], ref))
        report[family] = worst
        assert worst[True] <= 1.0, f"{family}: deterministic dw err/tol {worst[True]:.3g}"
        if family == "F1":
            assert worst[False] <= 1.0, f"F1: blocked-FP32 dw err/tol {worst[False]:.3g}"
    print(f"H{H} T{T} worst dw err/tol over 3 seeds: " +
          ", ".join(f"{f} det {r[True]:.3g} non-det {r[False]:.3g}" for f, r in report.items()))
