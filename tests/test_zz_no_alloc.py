"""rms_train_bwd_noalloc, the backward for callers that cannot allocate device memory
(allocator callbacks, runtimes with only pre-planned buffers, plugins whose host owns all
device memory): its scratch is a fixed array inside the library, so the caller passes
only inputs and outputs.  Checked through the C ABI against rms_train_bwd with a
caller-owned workspace, on two calls in a row (the second sees the array the first
left behind), within the tolerances of the other GPU tests.  This file is collected
last so a stop-at-first-failure run has already run everything else."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from bwd_rmsnorm_fwd_b200 import _lib, api, synth

from gpu_common import DW_ATOL, DW_RTOL, DX_ATOL, DX_RTOL, dev_rows, dev_weight

pytestmark = pytest.mark.gpu


def _call_noalloc(L, x, w, rstd, dy, dx, dw):
    T, H = x.shape
    rc = L.rms_train_bwd_noalloc(_lib.shape(T, 1, H), _lib.rows(x.data_ptr(), H, 0),
                                 w.data_ptr(), _lib.RMS_FP32 if w.dtype == torch.float32
                                 else _lib.RMS_BF16, rstd.data_ptr(),
                                 _lib.rows(dy.data_ptr(), H, 0), _lib.rows(dx.data_ptr(), H, 0),
                                 dw.data_ptr(), torch.cuda.current_stream().cuda_stream)
    _lib.check(rc)


@pytest.mark.parametrize("T,H,wdt", [(4099, 6144, "bf16"), (20000, 1536, "fp32"),
                                      (30000, 256, "bf16")])
def test_noalloc_backward_matches_the_workspace_backward(T, H, wdt):
    L = _lib.lib()
    x = dev_rows(synth.rows(21, "x", T, H))
    dy = dev_rows(synth.rows(21, "dy", T, H))
    w = dev_weight(synth.weight(21, H, wdt))
    _, rstd = api.rmsnorm_train_fwd(x, w)
    ref_dx, ref_dw = api.rmsnorm_train_bwd(x, w, rstd, dy, deterministic=False)
    torch.cuda.synchronize()
    assert api.bwd_path(T, 1, H, False) == 3   # the kernel that needs scratch
    for _ in range(2):
        dx = torch.full_like(x, float("nan"))
        dw = torch.full((H,), float("nan"), device="cuda")
        _call_noalloc(L, x, w, rstd, dy, dx, dw)
        torch.cuda.synchronize()
        a, b = dx.float(), ref_dx.float()
        assert torch.all((a - b).abs() <= DX_ATOL + DX_RTOL * b.abs())
        e = (dw.double() - ref_dw.double()).abs()
        assert torch.all(e <= DW_ATOL + DW_RTOL * ref_dw.double().abs())


def test_noalloc_rejects_widths_beyond_its_scratch():
    L = _lib.lib()
    rc = L.rms_train_bwd_noalloc(_lib.shape(4, 1, 8200), _lib.rows(1 << 20, 8200, 0), 1 << 21,
                                 0, 1 << 22, _lib.rows(1 << 23, 8200, 0),
                                 _lib.rows(1 << 24, 8200, 0), 1 << 25, None)
    assert rc == _lib.RMS_EINVAL
    assert b"8192" in L.rms_last_error()
