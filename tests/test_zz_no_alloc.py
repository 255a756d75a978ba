"""rms_train_bwd_noalloc, the backward for callers that cannot allocate device memory
(allocator callbacks, runtimes with only pre-planned buffers, plugins whose host owns all
device memory): its scratch is a fixed array inside the library, so the caller passes
only inputs and outputs.  Checked through the C ABI against rms_train_bwd with a
caller-owned workspace, on two calls in a row (the second sees the array the first
left behind), within the tolerances of the other GPU tests, and against the FP64 oracle.
This file is collected last so a stop-at-first-failure run has already run everything
else."""

from __future__ import annotations

import pytest
import torch

import oracle
from bwd_rmsnorm_fwd_b200 import _lib, api, synth

from gpu_common import (DW_ATOL, DW_RTOL, DX_ATOL, DX_RTOL, assert_dw, assert_dx, dev_rows,
                        dev_weight, host_bits)

pytestmark = pytest.mark.gpu


def _call_noalloc(L, x, w, rstd, dy, dx, dw):
    T, H = x.shape
    return L.rms_train_bwd_noalloc(_lib.shape(T, 1, H), _lib.rows(x.data_ptr(), H, 0),
                                   w.data_ptr(), _lib.RMS_FP32 if w.dtype == torch.float32
                                   else _lib.RMS_BF16, rstd.data_ptr(),
                                   _lib.rows(dy.data_ptr(), H, 0),
                                   _lib.rows(dx.data_ptr(), H, 0), dw.data_ptr(),
                                   torch.cuda.current_stream().cuda_stream)


# (T, H, weight dtype, backward program): the blocked-FP32 kernels (3) and the single-launch
# small-row kernel (1); both use the fixed array's ticket, accumulators and status word
CASES = [(4099, 6144, "bf16", 3), (20000, 1536, "fp32", 3), (30000, 256, "bf16", 3),
         (87, 2048, "bf16", 1), (1, 4096, "fp32", 1)]


@pytest.mark.parametrize("T,H,wdt,path", CASES)
def test_noalloc_backward_matches_the_workspace_backward(T, H, wdt, path):
    L = _lib.lib()
    xb, dyb = synth.rows(21, "x", T, H), synth.rows(21, "dy", T, H)
    wb = synth.weight(21, H, wdt)
    _, rstd_ref = oracle.train_fwd(xb, wb)
    dx_ref, dw_ref = oracle.train_bwd(xb, wb, rstd_ref, dyb)
    x, dy, w = dev_rows(xb), dev_rows(dyb), dev_weight(wb)
    rstd = torch.from_numpy(rstd_ref).cuda()
    ref_dx, ref_dw = api.rmsnorm_train_bwd(x, w, rstd, dy, deterministic=False)
    torch.cuda.synchronize()
    assert api.bwd_path(T, 1, H, False) == path
    for _ in range(2):
        dx = torch.full_like(x, float("nan"))
        dw = torch.full((H,), float("nan"), device="cuda")
        _lib.check(_call_noalloc(L, x, w, rstd, dy, dx, dw))
        _lib.check(L.rms_noalloc_status(torch.cuda.current_stream().cuda_stream))
        a, b = dx.float(), ref_dx.float()
        assert torch.all((a - b).abs() <= DX_ATOL + DX_RTOL * b.abs())
        e = (dw.double() - ref_dw.double()).abs()
        assert torch.all(e <= DW_ATOL + DW_RTOL * ref_dw.double().abs())
        assert_dx(host_bits(dx), dx_ref, f"noalloc dx {T}x{H}")
        assert_dw(dw.cpu().numpy(), dw_ref, f"noalloc dw {T}x{H}")


def test_noalloc_timeout_is_reported_and_the_next_call_is_correct():
    """A bounded wait that gives up (wait limit 0) sets the fixed array's status word; the
    word survives the calls after it until rms_noalloc_status reads and clears it, and
    calls after that are correct."""
    L = _lib.lib()
    T, H = 32768, 6144
    xb, dyb = synth.rows(22, "x", T, H), synth.rows(22, "dy", T, H)
    wb = synth.weight(22, H, "bf16")
    _, rstd_ref = oracle.train_fwd(xb, wb)
    _, dw_ref = oracle.train_bwd(xb, wb, rstd_ref, dyb, want_dx=False)
    x, dy, w = dev_rows(xb), dev_rows(dyb), dev_weight(wb)
    rstd = torch.from_numpy(rstd_ref).cuda()
    stream = torch.cuda.current_stream().cuda_stream
    dx = torch.empty_like(x)
    dw = torch.empty(H, device="cuda")
    assert api.bwd_path(T, 1, H, False) == 3
    _lib.check(L.rms_noalloc_status(stream))  # nothing pending
    prev = L.rms_set_wait_limit_cycles(0)
    try:
        _lib.check(_call_noalloc(L, x, w, rstd, dy, dx, dw))
        torch.cuda.synchronize()
    finally:
        L.rms_set_wait_limit_cycles(prev)
    _lib.check(_call_noalloc(L, x, w, rstd, dy, dx, dw))  # does not clear the word
    assert L.rms_noalloc_status(stream) == _lib.RMS_ETIMEOUT
    assert b"gave up" in L.rms_last_error()
    assert L.rms_noalloc_status(stream) == _lib.RMS_OK  # read and cleared
    for _ in range(2):
        _lib.check(_call_noalloc(L, x, w, rstd, dy, dx, dw))
        _lib.check(L.rms_noalloc_status(stream))
        assert_dw(dw.cpu().numpy(), dw_ref, "noalloc dw after a timeout")


def test_noalloc_rejects_widths_beyond_its_scratch():
    L = _lib.lib()
    rc = L.rms_train_bwd_noalloc(_lib.shape(4, 1, 8200), _lib.rows(1 << 20, 8200, 0), 1 << 21,
                                 0, 1 << 22, _lib.rows(1 << 23, 8200, 0),
                                 _lib.rows(1 << 24, 8200, 0), 1 << 25, None)
    assert rc == _lib.RMS_EINVAL
    assert b"8192" in L.rms_last_error()


def test_noalloc_rejected_call_then_valid_call():
    """A call that fails a host-side check (here dx overlapping dy) is rejected with its code
    before anything is queued; the next valid call is correct."""
    L = _lib.lib()
    T, H = 64, 512
    xb, dyb = synth.rows(23, "x", T, H), synth.rows(23, "dy", T, H)
    wb = synth.weight(23, H, "fp32")
    _, rstd_ref = oracle.train_fwd(xb, wb)
    dx_ref, dw_ref = oracle.train_bwd(xb, wb, rstd_ref, dyb)
    x, dy, w = dev_rows(xb), dev_rows(dyb), dev_weight(wb)
    rstd = torch.from_numpy(rstd_ref).cuda()
    dx = torch.empty_like(x)
    dw = torch.empty(H, device="cuda")
    assert _call_noalloc(L, x, w, rstd, dy, dy, dw) == _lib.RMS_EALIAS
    assert b"overlaps" in L.rms_last_error()
    _lib.check(_call_noalloc(L, x, w, rstd, dy, dx, dw))
    _lib.check(L.rms_noalloc_status(torch.cuda.current_stream().cuda_stream))
    assert_dx(host_bits(dx), dx_ref, "noalloc dx after a rejected call")
    assert_dw(dw.cpu().numpy(), dw_ref, "noalloc dw after a rejected call")
