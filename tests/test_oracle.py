"""Pins of the FP64 oracle against facts that do not come from the oracle itself:
closed forms, finite differences of the forward, algebraic identities, exact
rational sums, the pages' cancellation example, torch's own BF16 conversion, and
brute force in exact rational arithmetic.  No GPU needed."""

from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from bwd_rmsnorm_fwd_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bits_of(vals) -> np.ndarray:
    """BF16 bits of values that are exactly representable in BF16 (checked)."""
    f = np.asarray(vals, dtype=np.float32)
    b = synth.f32_to_bf16_bits(f)
    assert np.array_equal(synth.bf16_bits_to_f32(b), f), "value not exactly BF16"
    return b


def frac_to_bf16_bits(q: Fraction) -> int:
    """Exact rational -> BF16 bits, nearest-even (normal range only; test helper)."""
    if q == 0:
        return 0
    neg = q < 0
    a = -q if neg else q
    e = math.floor(math.log2(a))
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    quantum = Fraction(2) ** (e - 7)
    n = a / quantum
    k = math.floor(n)
    rem = n - k
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and k % 2 == 1):
        k += 1
    val = float(k * quantum)
    b = int(np.array([val], np.float32).view(np.uint32)[0] >> 16)
    return b | (0x8000 if neg else 0)


# ---- BF16 conversion -----------------------------------------------------------------

def test_bf16_rounding_matches_torch_on_fp32_values(oracle_mod):
    g = np.random.default_rng(1)
    v = (g.standard_normal(20000) * np.exp2(g.integers(-140, 120, 20000))).astype(np.float32)
    v = v[np.isfinite(v)]
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle_mod.bf16_from_f64(v.astype(np.float64))
    assert np.array_equal(got, ref)


def test_bf16_ties_edges_and_single_rounding(oracle_mod):
    cases = [
        (1.0 + 2.0 ** -8, 0x3F80),                 # tie -> even (1.0)
        (1.0 + 3 * 2.0 ** -8, 0x3F82),             # tie -> even (1 + 2^-6)
        (-(1.0 + 2.0 ** -8), 0xBF80),
        (1.0 + 2.0 ** -8 + 2.0 ** -40, 0x3F81),    # above the tie: a double->float->bf16
                                                   # chain would round this down to 1.0
        (2.0 ** -133, 0x0001),                     # smallest subnormal
        (2.0 ** -134, 0x0000),                     # tie between 0 and 2^-133 -> even (0)
        (3 * 2.0 ** -135, 0x0001),
        ((2 - 2.0 ** -7) * 2.0 ** 127, 0x7F7F),    # largest finite
        ((2 - 2.0 ** -8) * 2.0 ** 127, 0x7F80),    # overflow threshold (tie) -> inf
        ((2 - 2.0 ** -8) * 2.0 ** 127 * (1 - 2.0 ** -30), 0x7F7F),
        (float("inf"), 0x7F80),
        (0.0, 0x0000),
        (-0.0, 0x8000),
    ]
    got = oracle_mod.bf16_from_f64(np.array([c[0] for c in cases]))
    assert [int(b) for b in got] == [c[1] for c in cases]
    assert oracle_mod.bf16_from_f64(np.array([float("nan")]))[0] == 0x7FC0


# ---- forward closed forms ------------------------------------------------------------------

@pytest.mark.parametrize("wdt", ["bf16", "fp32"])
def test_fwd_power_of_two_rows(oracle_mod, wdt):
    """Rows of +-2^k with eps = 0: mean(x^2) = 4^k, so rstd = 2^-k and y = sign * w exactly."""
    g = np.random.default_rng(2)
    R, H = 12, 40
    k = g.integers(-20, 20, R)
    sign = np.where(g.random((R, H)) < 0.5, -1.0, 1.0)
    x = bits_of(sign * np.exp2(k)[:, None])
    w = synth.weight(3, H, wdt)
    y, rstd = oracle_mod.train_fwd(x, w, eps=0.0)
    assert np.array_equal(rstd, np.exp2(-k).astype(np.float32))
    wf = synth.bf16_bits_to_f32(w) if wdt == "bf16" else w
    expect = synth.f32_to_bf16_bits((sign * wf[None, :]).astype(np.float32))
    assert np.array_equal(y, expect)


def test_fwd_eps_is_added_to_the_mean(oracle_mod):
    """H = 4, x = +-2, eps = 12: mean(x^2) + eps = 16, so rstd = 1/4 exactly.  (eps added
    to the sum, or outside the square root, gives a different value.)"""
    x = bits_of([[2.0, -2.0, 2.0, 2.0]])
    w = bits_of([1.0, 0.5, -3.0, 1.25])
    y, rstd, rstd64 = oracle_mod.train_fwd(x, w, eps=12.0, want_rstd64=True)
    assert rstd64[0] == 0.25 and rstd[0] == np.float32(0.25)
    assert np.array_equal(y, bits_of([[0.5, -0.25, -1.5, 0.625]]))


def test_fwd_constant_row(oracle_mod):
    """A constant row c (eps = 0) normalises to sign(c): y = sign(c) * w."""
    x = bits_of(np.full((2, 16), [[-3.0], [0.375]]))
    w = synth.weight(5, 16, "fp32")
    y, rstd, rstd64 = oracle_mod.train_fwd(x, w, eps=0.0, want_rstd64=True)
    assert np.allclose(rstd64, [1 / 3.0, 1 / 0.375], rtol=1e-15)
    expect = synth.f32_to_bf16_bits(np.stack([-w, w]).astype(np.float32))
    assert np.array_equal(y, expect)


def test_fwd_scale_invariance(oracle_mod):
    """eps = 0: y(2^m x) == y(x) bit for bit and rstd scales by 2^-m exactly."""
    x = synth.rows(7, "x", 16, 96, "F1")
    w = synth.weight(7, 96, "bf16")
    y0, r0 = oracle_mod.train_fwd(x, w, eps=0.0)
    x8 = bits_of(synth.bf16_bits_to_f32(x) * np.float32(256.0))
    y1, r1 = oracle_mod.train_fwd(x8, w, eps=0.0)
    assert np.array_equal(y0, y1)
    assert np.array_equal(r1, (r0 / np.float32(256.0)).astype(np.float32))


# ---- backward: derivatives of the forward ----------------------------------------------

def _fd_loss(oracle_mod, x, w, dy, eps, dh=None):
    y, _ = oracle_mod.fwd_f64(x, w, eps)
    L = float(np.sum(dy * y))
    if dh is not None:
        L += float(np.sum(dh * x))
    return L


@pytest.mark.parametrize("residual", [False, True])
def test_backward_is_the_gradient_of_the_forward(oracle_mod, residual):
    """Central finite differences of L = sum(dy * y(x, w)) (+ sum(dh * x) for the residual
    form, whose backward returns dL/dh) against the oracle's dx and dw."""
    g = np.random.default_rng(11)
    R, H, eps = 3, 6, 1e-3
    x = g.standard_normal((R, H))
    w = 1 + 0.1 * g.standard_normal(H)
    dy = g.standard_normal((R, H))
    dh = g.standard_normal((R, H)) if residual else None
    _, rstd = oracle_mod.fwd_f64(x, w, eps)
    dx, dw = oracle_mod.bwd_f64(x, w, rstd, dy, dh)
    step = 1e-6
    for r in range(R):
        for j in range(H):
            xp, xm = x.copy(), x.copy()
            xp[r, j] += step
            xm[r, j] -= step
            fd = (_fd_loss(oracle_mod, xp, w, dy, eps, dh) -
                  _fd_loss(oracle_mod, xm, w, dy, eps, dh)) / (2 * step)
            assert abs(fd - dx[r, j]) <= 1e-7 * max(1.0, abs(fd)), (r, j, fd, dx[r, j])
    for j in range(H):
        wp, wm = w.copy(), w.copy()
        wp[j] += step
        wm[j] -= step
        fd = (_fd_loss(oracle_mod, x, wp, dy, eps, dh) -
              _fd_loss(oracle_mod, x, wm, dy, eps, dh)) / (2 * step)
        assert abs(fd - dw[j]) <= 1e-7 * max(1.0, abs(fd)), (j, fd, dw[j])


@pytest.mark.parametrize("eps", [0.0, 1e-6, 0.25])
def test_dx_dot_x_identity(oracle_mod, eps):
    """sum_j dx_j x_j = eps * rstd^3 * sum_j dy_j w_j x_j for rstd = 1/sqrt(mean x^2 + eps);
    with eps = 0 this is the scale invariance of the forward (dx orthogonal to x)."""
    x = synth.bf16_bits_to_f32(synth.rows(21, "x", 8, 64)).astype(np.float64)
    dy = synth.bf16_bits_to_f32(synth.rows(21, "dy", 8, 64)).astype(np.float64)
    w = synth.weight(21, 64, "fp32").astype(np.float64)
    rstd = 1.0 / np.sqrt(np.mean(x * x, axis=1) + eps)
    dx, _ = oracle_mod.bwd_f64(x, w, rstd, dy)
    lhs = np.sum(dx * x, axis=1)
    rhs = eps * rstd ** 3 * np.sum(dy * w * x, axis=1)
    scale = np.sum(np.abs(dx * x), axis=1)
    assert np.all(np.abs(lhs - rhs) <= 1e-12 * scale + 1e-300)


def test_h1_is_the_textbook_derivative(oracle_mod):
    """H = 1: y = w x / sqrt(x^2 + eps), so dy/dx = w eps / (x^2 + eps)^(3/2)."""
    x = np.array([[0.3], [-2.0], [1e-3], [7.5]])
    w = np.array([1.7])
    dy = np.array([[1.0], [-0.5], [2.0], [0.25]])
    eps = 0.01
    _, rstd = oracle_mod.fwd_f64(x, w, eps)
    dx, dw = oracle_mod.bwd_f64(x, w, rstd, dy)
    expect_dx = dy[:, 0] * w[0] * eps / (x[:, 0] ** 2 + eps) ** 1.5
    # g - xh*c = g (1 - xh^2) cancels by up to eps / x^2 ~ 2e-4 here: allow ~1e4 ulps
    assert np.allclose(dx[:, 0], expect_dx, rtol=1e-11, atol=0)
    expect_dw = np.sum(dy[:, 0] * x[:, 0] / np.sqrt(x[:, 0] ** 2 + eps))
    assert math.isclose(dw[0], expect_dw, rel_tol=1e-13)


# ---- dw: exact sums ---------------------------------------------------------------------------

def test_dw_exact_integer_sums(oracle_mod):
    """Rows of +-2^k with eps = 0 give x*rstd = +-1 exactly; integer dy then makes every dw
    column an exact integer sum, computed here with Python integers."""
    g = np.random.default_rng(4)
    R, H = 300, 24
    k = g.integers(-6, 7, R)
    sign = np.where(g.random((R, H)) < 0.5, -1, 1)
    x = bits_of(sign * np.exp2(k)[:, None])
    dyi = g.integers(-256, 257, (R, H))
    dy = bits_of(dyi)
    w = synth.weight(4, H, "bf16")
    _, rstd = oracle_mod.train_fwd(x, w, eps=0.0)
    _, dw = oracle_mod.train_bwd(x, w, rstd, dy, want_dx=False)
    exact = [sum(int(sign[r, j]) * int(dyi[r, j]) for r in range(R)) for j in range(H)]
    assert [float(v) for v in dw] == [float(e) for e in exact]


def test_dw_and_dx_against_exact_rationals(oracle_mod):
    """Brute force in exact rational arithmetic on BF16 inputs and FP32 rstd: dw to within
    one FP64 rounding per row, dx (unrounded) to 1e-13 relative and BF16 dx bit-exact
    except where the exact value sits within 1e-12 of a rounding tie."""
    R, H = 5, 7
    x = synth.rows(31, "x", R, H)
    dy = synth.rows(31, "dy", R, H)
    w = synth.weight(31, H, "fp32")
    rstd = np.array([0.83, 1.21, 0.5, 2.0, 0.97], np.float32)
    dxb, dw = oracle_mod.train_bwd(x, w, rstd, dy)
    X = [[Fraction(float(v)) for v in row] for row in synth.bf16_bits_to_f32(x)]
    D = [[Fraction(float(v)) for v in row] for row in synth.bf16_bits_to_f32(dy)]
    W = [Fraction(float(v)) for v in w]
    S = [Fraction(float(v)) for v in rstd]
    for j in range(H):
        exact = sum(D[r][j] * X[r][j] * S[r] for r in range(R))
        bound = R * 2.0 ** -52 * float(sum(abs(D[r][j] * X[r][j] * S[r]) for r in range(R)))
        assert abs(float(exact) - dw[j]) <= bound
    for r in range(R):
        xh = [X[r][j] * S[r] for j in range(H)]
        gg = [D[r][j] * W[j] for j in range(H)]
        c = sum(a * b for a, b in zip(gg, xh)) / H
        for j in range(H):
            exact = S[r] * (gg[j] - xh[j] * c)
            b = frac_to_bf16_bits(exact)
            if int(dxb[r, j]) != b:
                # only acceptable right at a tie of the BF16 grid
                e = math.floor(math.log2(abs(float(exact))))
                q = Fraction(2) ** (e - 7)
                frac_part = (abs(exact) / q) % 1
                assert abs(frac_part - Fraction(1, 2)) < Fraction(1, 10 ** 12), (r, j)


def test_cancellation_example_from_the_pages(oracle_mod):
    """The review example (65536, 2^-10, -65536 in row order): exact sum 2^-10; a plain FP32
    running sum returns 0, which the dw budget (atol 1e-4 + rtol 1e-4) rejects."""
    fields = {}
    with open(os.path.join(GOLDEN, "cancellation_products.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                k, *v = line.split()
                fields[k] = [float(t) for t in v]
    prods = fields["products"]
    exact = fields["exact_sum"][0]
    H = 8
    x = bits_of(np.ones((len(prods), H)))           # rstd = 1, x*rstd = 1 exactly (eps = 0)
    dy = bits_of(np.repeat(np.array(prods)[:, None], H, axis=1))
    w = synth.weight(0, H, "fp32")
    _, rstd = oracle_mod.train_fwd(x, w, eps=0.0)
    assert np.all(rstd == 1.0)
    _, dw = oracle_mod.train_bwd(x, w, rstd, dy, want_dx=False)
    assert np.all(dw == exact)
    run = np.float32(0.0)
    for p in prods:
        run = np.float32(run + np.float32(p))
    assert float(run) == fields["fp32_running_sum"][0]
    assert abs(float(run) - exact) > 1e-4 + 1e-4 * abs(exact)


# ---- residual form ---------------------------------------------------------------------------

def test_residual_h_is_the_bf16_sum(oracle_mod):
    """h = BF16(x + residual), checked against torch's BF16 addition (FP32 add of two BF16
    values is exact whenever it can matter, then one nearest-even rounding)."""
    R, H = 64, 256
    x = synth.rows(8, "x", R, H)
    res = synth.rows(8, "res", R, H)
    w = synth.weight(8, H, "bf16")
    h, y, rstd = oracle_mod.train_fwd(x, w, eps=1e-6, residual=res)
    tx = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16)
    tr = torch.from_numpy(res.view(np.int16)).view(torch.bfloat16)
    ref = (tx.float() + tr.float()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(h, ref)
    y2, rstd2 = oracle_mod.train_fwd(h, w, eps=1e-6)
    assert np.array_equal(y, y2) and np.array_equal(rstd, rstd2)


def test_residual_bwd_adds_dh(oracle_mod):
    """grad_h = BF16(dh + dx_formula): with dy = 0 the norm's gradient vanishes, so
    grad_h == dh bit for bit."""
    R, H = 16, 64
    h = synth.rows(9, "x", R, H)
    dh = synth.rows(9, "dh", R, H)
    dy = np.zeros((R, H), np.uint16)
    w = synth.weight(9, H, "bf16")
    _, rstd = oracle_mod.train_fwd(h, w)
    gh, dw = oracle_mod.train_bwd(h, w, rstd, dy, dh=dh)
    assert np.array_equal(gh, dh)
    assert np.all(dw == 0)


# ---- housekeeping -------------------------------------------------------------------------

def test_thread_count_does_not_change_bits(oracle_mod):
    R, H = 257, 136
    x = synth.rows(5, "x", R, H, "F2")
    dy = synth.rows(5, "dy", R, H, "F2")
    w = synth.weight(5, H, "fp32")
    a = oracle_mod.train_fwd(x, w, nthreads=1)
    b = oracle_mod.train_fwd(x, w, nthreads=7)
    assert all(np.array_equal(p, q) for p, q in zip(a, b))
    da = oracle_mod.train_bwd(x, w, a[1], dy, nthreads=1)
    db = oracle_mod.train_bwd(x, w, a[1], dy, nthreads=5)
    assert np.array_equal(da[0], db[0]) and np.array_equal(da[1], db[1])


def test_input_families_have_their_structure():
    x = synth.bf16_bits_to_f32(synth.rows(1, "x", 4096, 64, "F3"))
    dy = synth.bf16_bits_to_f32(synth.rows(1, "dy", 4096, 64, "F3"))
    assert np.array_equal(x[0::2], x[1::2])
    rel = np.abs(dy[1::2] + dy[0::2]) / np.maximum(np.abs(dy[0::2]), 1e-30)
    assert np.median(rel) < 2 ** -7
    x2 = synth.bf16_bits_to_f32(synth.rows(1, "x", 4096, 64, "F2"))
    assert np.max(np.abs(x2)) > 100
    # rows regenerate identically from any offset
    full = synth.rows(3, "dy", 3000, 32)
    assert np.array_equal(full[1500:2100], synth.rows(3, "dy", 3000, 32, row0=1500, nrows=600))
    assert np.array_equal(full[[5, 2999, 1024]], synth.sample_rows(3, "dy", 3000, 32,
                                                                 [5, 2999, 1024]))


def test_strided_layout_round_trip():
    T, heads, H, st, sk = 5, 3, 16, 96, 32
    rows = synth.rows(2, "x", T * heads, H)
    buf = synth.place_rows(rows, T, heads, H, st, sk)
    assert buf.size == synth.view_extent(T, heads, H, st, sk)
    assert np.array_equal(synth.gather_rows(buf, T, heads, H, st, sk), rows)
    # untouched gap elements keep the fill pattern
    assert buf[H] == 0x7FC1
