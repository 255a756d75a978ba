"""Gradient accumulation (dw += the call's sum) and the autograd wrapper, through the C ABI.

Accumulation is defined as dw = FP32(dw_prev + dw_call), dw_call being exactly what the
overwrite call returns: the deterministic mode is checked bit for bit against that FP32 sum
computed on the host, both modes against dw_prev + the FP64 oracle within the dw budget.  The
autograd function is checked against the oracle (dx, dw; the residual form's gradient of h
reaching both x and residual), with a float32 main-grad buffer accumulated over
micro-batches, and under activation checkpointing (the pages' 2xfwd+bwd step), where the
recomputed forward gives the same bits."""

from __future__ import annotations

import numpy as np
import pytest
import torch
from torch.utils.checkpoint import checkpoint

import oracle
from bwd_rmsnorm_fwd_b200 import api, synth

from gpu_common import assert_dw, assert_dx, dev_rows, dev_weight, host_bits

pytestmark = pytest.mark.gpu


def _inputs(T, H, wdt, seed, residual=False):
    x = synth.rows(seed, "x", T, H)
    dy = synth.rows(seed, "dy", T, H)
    w = synth.weight(seed, H, wdt)
    res = synth.rows(seed, "res", T, H) if residual else None
    dh = synth.rows(seed, "dh", T, H) if residual else None
    return x, dy, w, res, dh


# (T, H, w dtype, residual): single-launch program, deterministic pair / blocked FP32 staged,
# blocked FP32 one-warp-per-row, residual form
ACC_CASES = [(87, 2048, "bf16", False), (4099, 6144, "fp32", False), (20000, 256, "bf16", False),
             (3000, 1536, "bf16", True)]


@pytest.mark.parametrize("det", [True, False])
@pytest.mark.parametrize("T,H,wdt,residual", ACC_CASES)
def test_accumulate_adds_the_overwrite_result(T, H, wdt, residual, det):
    x, dy, w, res, dh = _inputs(T, H, wdt, 31, residual)
    if residual:
        h, _, rstd = oracle.train_fwd(x, w, residual=res)
    else:
        h = x
        _, rstd = oracle.train_fwd(x, w)
    dx_ref, dw_ref = oracle.train_bwd(h, w, rstd, dy, dh=dh)
    hd, dyd, wd = dev_rows(h), dev_rows(dy), dev_weight(w)
    dhd = dev_rows(dh) if residual else None
    rs = torch.from_numpy(rstd).cuda()
    prev = np.random.default_rng(T + H).standard_normal(H).astype(np.float32) * 4
    _, dw0 = api.rmsnorm_train_bwd(hd, wd, rs, dyd, deterministic=det, dh=dhd)
    dw0 = dw0.cpu().numpy()
    acc = torch.from_numpy(prev.copy()).cuda()
    dx, _ = api.rmsnorm_train_bwd(hd, wd, rs, dyd, deterministic=det, dh=dhd, dw=acc,
                                  accumulate=True)
    api.status()
    got = acc.cpu().numpy()
    assert_dx(host_bits(dx), dx_ref, "dx of the accumulating call")
    assert_dw(got, prev.astype(np.float64) + dw_ref, f"accumulated dw det={det}")
    if det:
        want = (prev + dw0).astype(np.float32)  # one FP32 addition, nearest-even
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
        # a second accumulation adds the same bits again
        api.rmsnorm_train_bwd(hd, wd, rs, dyd, deterministic=True, dh=dhd, dw=acc,
                              accumulate=True)
        want2 = (want + dw0).astype(np.float32)
        assert np.array_equal(acc.cpu().numpy().view(np.uint32), want2.view(np.uint32))


def test_accumulate_with_no_rows_leaves_dw():
    H = 512
    w = dev_weight(synth.weight(0, H, "fp32"))
    x = torch.empty(0, H, dtype=torch.bfloat16, device="cuda")
    rstd = torch.empty(0, device="cuda")
    acc = torch.arange(H, dtype=torch.float32, device="cuda")
    api.rmsnorm_train_bwd(x, w, rstd, x, dw=acc, accumulate=True)
    torch.cuda.synchronize()
    assert torch.equal(acc, torch.arange(H, dtype=torch.float32, device="cuda"))


@pytest.mark.parametrize("wdt", ["fp32", "bf16"])
@pytest.mark.parametrize("det", [True, False])
def test_autograd_matches_the_oracle(det, wdt):
    T, H = 3000, 2048
    x, dy, w, _, _ = _inputs(T, H, wdt, 32)
    _, rstd = oracle.train_fwd(x, w)
    dx_ref, dw_ref = oracle.train_bwd(x, w, rstd, dy)
    xd = dev_rows(x).requires_grad_(True)
    wd = dev_weight(w).requires_grad_(True)
    y = api.rmsnorm_train(xd, wd, deterministic=det)
    y.backward(dev_rows(dy))
    api.status()
    assert_dx(host_bits(xd.grad), dx_ref, "autograd dx")
    assert wd.grad.dtype == wd.dtype
    if wdt == "fp32":
        assert_dw(wd.grad.cpu().numpy(), dw_ref, "autograd dw")
    else:  # autograd rounds the FP32 dw to the BF16 weight's dtype
        g = wd.grad.float().cpu().numpy().astype(np.float64)
        assert np.all(np.abs(g - dw_ref) <= 2.0 ** -8 * np.abs(dw_ref) + 1e-4)


def test_autograd_main_grad_accumulates_micro_batches():
    """Two micro-batches through the autograd function with a float32 main-grad buffer: the
    buffer ends as FP32(FP32(0 + dw_1) + dw_2) in deterministic mode (dw_i from the plain
    overwrite backward), within the budget of the summed FP64 oracle, and w gets no gradient
    of its own."""
    T, H = 2500, 1536
    wb = synth.weight(33, H, "bf16")
    wd = dev_weight(wb).requires_grad_(True)
    main = torch.zeros(H, dtype=torch.float32, device="cuda")
    want = np.zeros(H, np.float32)
    ref64 = np.zeros(H)
    for mb in range(2):
        x, dy, _, _, _ = _inputs(T, H, "bf16", 40 + mb)
        _, rstd = oracle.train_fwd(x, wb)
        _, dw_ref = oracle.train_bwd(x, wb, rstd, dy, want_dx=False)
        ref64 += dw_ref
        xd = dev_rows(x).requires_grad_(True)
        y = api.rmsnorm_train(xd, wd, deterministic=True, main_grad=main)
        y.backward(dev_rows(dy))
        _, rs_gpu = api.rmsnorm_train_fwd(xd.detach(), wd.detach())
        _, dw_plain = api.rmsnorm_train_bwd(xd.detach(), wd.detach(), rs_gpu, dev_rows(dy),
                                            deterministic=True)
        want = (want + dw_plain.cpu().numpy()).astype(np.float32)
    api.status()
    assert wd.grad is None
    assert np.array_equal(main.cpu().numpy().view(np.uint32), want.view(np.uint32))
    assert_dw(main.cpu().numpy(), ref64, "main_grad over two micro-batches")


@pytest.mark.parametrize("det", [True, False])
def test_checkpointed_step_gives_the_same_gradients(det):
    """The pages' checkpointed step (forward, forward recomputed in the backward, backward)
    under torch.utils.checkpoint: the recomputed forward reproduces rstd bit for bit, so the
    gradients equal those of the uncheckpointed call (bit for bit in deterministic mode)."""
    T, H = 4096, 6144
    x, dy, w, _, _ = _inputs(T, H, "fp32", 34)
    dyd = dev_rows(dy)
    grads = []
    for ckpt in (False, True):
        xd = dev_rows(x).requires_grad_(True)
        wd = dev_weight(w).requires_grad_(True)
        if ckpt:
            y = checkpoint(api.rmsnorm_train, xd, wd, 1e-6, None, det, use_reentrant=False)
        else:
            y = api.rmsnorm_train(xd, wd, 1e-6, None, det)
        y.backward(dyd)
        grads.append((host_bits(xd.grad), wd.grad.cpu().numpy()))
    api.status()
    assert np.array_equal(grads[0][0], grads[1][0])
    if det:
        assert np.array_equal(grads[0][1].view(np.uint32), grads[1][1].view(np.uint32))
    _, rstd = oracle.train_fwd(x, w)
    dx_ref, dw_ref = oracle.train_bwd(x, w, rstd, dy)
    assert_dx(grads[1][0], dx_ref, "checkpointed dx")
    assert_dw(grads[1][1], dw_ref, "checkpointed dw")


def test_residual_autograd_sends_grad_h_to_x_and_residual():
    T, H = 2000, 6144
    x, dy, w, res, dh = _inputs(T, H, "bf16", 35, residual=True)
    h, y_ref, rstd = oracle.train_fwd(x, w, residual=res)
    gh_ref, dw_ref = oracle.train_bwd(h, w, rstd, dy, dh=dh)
    xd = dev_rows(x).requires_grad_(True)
    rd = dev_rows(res).requires_grad_(True)
    wd = dev_weight(w).requires_grad_(True)
    y, hd = api.rmsnorm_train(xd, wd, residual=rd, deterministic=True)
    assert np.array_equal(host_bits(hd), h)
    torch.autograd.backward([y, hd], [dev_rows(dy), dev_rows(dh)])
    api.status()
    assert_dx(host_bits(xd.grad), gh_ref, "grad of x")
    assert np.array_equal(host_bits(xd.grad), host_bits(rd.grad))
    g = wd.grad.float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(g - dw_ref) <= 2.0 ** -8 * np.abs(dw_ref) + 1e-4)
