"""Failure detection without a GPU fault: the backward's pipeline waits are bounded.  With
the limit set to zero cycles the first wait that is not already satisfied gives up; the
kernel records RMS_ETIMEOUT in the workspace status word, stops waiting, lets its bulk
copies land and returns.  The host reads the status, and the next call on the same
context and workspace is correct."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from bwd_rmsnorm_fwd_b200 import _lib, api, synth

from gpu_common import assert_dw, dev_rows, dev_weight

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("det", [False, True])
def test_wait_limit_reports_timeout_and_context_survives(det):
    T, H = 32768, 6144
    x = synth.rows(13, "x", T, H)
    dy = synth.rows(13, "dy", T, H)
    w = synth.weight(13, H, "bf16")
    _, rstd = oracle.train_fwd(x, w)
    _, dw_ref = oracle.train_bwd(x, w, rstd, dy, want_dx=False)
    xd, dyd, wd, rs = dev_rows(x), dev_rows(dy), dev_weight(w), torch.from_numpy(rstd).cuda()
    ws = api.Workspace("cuda")
    L = _lib.lib()
    assert api.bwd_path(T, 1, H, det) in (2, 3)
    prev = L.rms_set_wait_limit_cycles(0)
    try:
        api.rmsnorm_train_bwd(xd, wd, rs, dyd, deterministic=det, workspace=ws)
        torch.cuda.synchronize()
    finally:
        L.rms_set_wait_limit_cycles(prev)
    with pytest.raises(_lib.RmsError) as ei:
        api.status(ws)
    assert ei.value.code == _lib.RMS_ETIMEOUT
    api.status(ws)  # the word was cleared
    for _ in range(2):
        _, dw = api.rmsnorm_train_bwd(xd, wd, rs, dyd, deterministic=det, workspace=ws)
        api.status(ws)
        assert_dw(dw.cpu().numpy(), dw_ref, f"after timeout det={det}")


def test_forward_has_no_waits_to_time_out():
    """The forward kernels never wait on the device: with the wait limit at zero cycles the
    forward still completes, correct, and its status check stays clean."""
    T, H = 32768, 6144
    x = synth.rows(14, "x", T, H)
    w = synth.weight(14, H, "fp32")
    y_ref, rstd_ref = oracle.train_fwd(x, w)
    xd, wd = dev_rows(x), dev_weight(w)
    L = _lib.lib()
    prev = L.rms_set_wait_limit_cycles(0)
    try:
        y, rstd = api.rmsnorm_train_fwd(xd, wd)
        api.forward_status()
    finally:
        L.rms_set_wait_limit_cycles(prev)
    from gpu_common import assert_fwd, host_bits
    assert_fwd(host_bits(y), rstd.cpu().numpy(), y_ref, rstd_ref, "forward at wait limit 0")
