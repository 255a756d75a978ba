"""The deterministic dw order checked on the CPU, independently of any GPU run.

* The order's IEEE emulation meets the dw budget (per element atol 1e-4 + rtol 1e-4 against
  FP64, flashinfer PR #8848 "Measurement") at the plans the library picks for the pages'
  shapes, on all three input families.
* On rows of +-2^k with eps = 0, rstd = 2^-k and xh = +-1 exactly, so dw_j is an exact dyadic
  sum.  Every plan must then reproduce it bit for bit: blocks, chunk folds and segment folds
  add no error where there is none to add (PR #8512 introduction: exact products, TwoSum).

The plan (B, L, S) comes from the library's host-side query; nothing here needs a GPU."""

from __future__ import annotations

import numpy as np
import pytest

import oracle
from bwd_rmsnorm_fwd_b200 import api, build, synth

from det_order import emulate_det_dw
from gpu_common import dw_ratio


@pytest.fixture(scope="module", autouse=True)
def _library():
    build.build()


@pytest.mark.parametrize("T,heads,H,family", [(2048, 1, 512, "F1"), (5000, 1, 1536, "F2"),
                                              (700, 24, 256, "F3"), (33000, 1, 264, "F1"),
                                              (4100, 1, 2048, "F3")])
def test_order_meets_the_dw_budget(T, heads, H, family):
    R = T * heads
    x = synth.rows(11, "x", R, H, family)
    dy = synth.rows(11, "dy", R, H, family)
    w = synth.weight(11, H, "bf16")
    _, rstd = oracle.train_fwd(x, w)
    _, ref = oracle.train_bwd(x, w, rstd, dy, want_dx=False)
    B, L, S = api.det_plan(T, heads, H)
    got = emulate_det_dw(x, dy, rstd, B, L, S)
    r = dw_ratio(got, ref)
    print(f"T{T} heads{heads} H{H} {family} plan {(B, L, S)}: dw err/tol {r:.3g}")
    assert r <= 1.0


def test_order_reproduces_exact_sums_bit_for_bit():
    R, H = 3000, 64
    rng = np.random.default_rng(3)
    k = rng.integers(-3, 4, size=R)
    sign = rng.choice([-1.0, 1.0], size=(R, H))
    x = synth.f32_to_bf16_bits((sign * (2.0 ** k)[:, None]).astype(np.float32))
    dyv = rng.integers(-64, 65, size=(R, H)) / 8.0          # exact in BF16
    dy = synth.f32_to_bf16_bits(dyv.astype(np.float32))
    w = np.ones(H, np.float32)
    _, rstd = oracle.train_fwd(x, w, 0.0)
    assert np.array_equal(rstd, (2.0 ** -k).astype(np.float32))
    exact = (sign * dyv).sum(axis=0)                        # dyadic, exact in FP64 and FP32
    _, ref = oracle.train_bwd(x, w, rstd, dy, want_dx=False)
    assert np.array_equal(ref, exact)
    for B, L, S in [(16, 16, 16), (8, 4, 16), (64, 1, 16), (32, 2, 16), api.det_plan(R, 1, H)]:
        got = emulate_det_dw(x, dy, rstd, B, L, S)
        assert np.array_equal(got, exact.astype(np.float32)), (B, L, S)
