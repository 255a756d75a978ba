// Oracle for training RMSNorm (forward, backward, residual form) -- TEST INFRASTRUCTURE ONLY.
//
// This file is the slow, plain, obviously-correct CPU definition that the CUDA
// path is checked against.  Only the tests, the smoke check and the benchmark's
// CPU-baseline leg may load it; the product library never does, and the two
// share no code, headers or constants.
//
// Everything is computed in IEEE double from the exact BF16 / FP32 input bits;
// outputs are rounded once, the way the public API returns them (BF16 with
// round-to-nearest-even, FP32 with round-to-nearest-even).
//
// What is computed (sources: the pages "fix(cake_rmsnorm_det): fixed-order dw for
// the smallest token counts of the SM100/SM103 backward" (flashinfer PR #8512) and
// "...sm_100a non-deterministic backward..." (flashinfer PR #8848), their
// introductions and the "Measurement" / "Key" sections):
//   forward      rstd_r = 1 / sqrt(mean_j(x_rj^2) + eps),  y_rj = x_rj * rstd_r * w_j
//                y is BF16, rstd FP32 (PR #8848 introduction; "Workload: eps 1e-6").
//   residual     h_rj = BF16(x_rj + residual_rj); the forward above runs on h; h is
//                returned (PR #8512 introduction, "Residual rows"; PR #8848 "Key":
//                h_new = BF16(h + u)).
//   backward     with xh = x * rstd, g = dy * w, c_r = (1/H) sum_j g_rj xh_rj:
//                dx_rj = rstd_r (g_rj - xh_rj c_r)            (BF16)
//                dw_j  = sum_r dy_rj x_rj rstd_r              (FP32 on the API; kept
//                                                              in FP64 here)
//                this is the gradient of sum(dy * y) for the forward above; the
//                backward uses the FP32 rstd the forward returned.
//   residual bwd grad_h = BF16(dh + dx_formula): the backward takes the gradients of
//                y and of h and returns the gradient of h (PR #8512 "Residual rows").
//
// Threads: rows are split across threads for the row outputs; dw columns are split
// across threads and every column is summed in increasing row order, so the
// result does not depend on the thread count.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>
#include <algorithm>

namespace {

// ---- BF16 <-> double, written from the IEEE-754 definition -------------------------

double bf16_to_double(uint16_t b) {
    uint32_t u = static_cast<uint32_t>(b) << 16;  // a BF16 value is the top half of an FP32
    float f;
    std::memcpy(&f, &u, 4);
    return static_cast<double>(f);
}

// Correctly rounded (nearest, ties to even) conversion of a double to BF16:
// 8 significant bits, FP32's exponent range, gradual underflow, overflow to inf.
uint16_t double_to_bf16(double v) {
    if (std::isnan(v)) return 0x7FC0;
    const bool neg = std::signbit(v);
    double a = std::fabs(v);
    double r;
    if (a == 0.0) {
        r = 0.0;
    } else {
        int E;
        std::frexp(a, &E);          // a = m * 2^E, m in [0.5, 1)
        int e = E - 1;              // a = (2m) * 2^e, 2m in [1, 2)
        if (e < -126) e = -126;     // subnormal BF16 values share the quantum 2^-133
        const double q = std::ldexp(1.0, e - 7);   // spacing of BF16 values near a
        const double n = a / q;                    // exact: q is a power of two
        const double k = std::nearbyint(n);        // default rounding mode: ties to even
        r = k * q;                                 // exact; may be 2^(e+1) (next binade)
    }
    float f = static_cast<float>(r);               // exact, or inf when r >= 2^128
    uint32_t u;
    std::memcpy(&u, &f, 4);
    uint16_t b = static_cast<uint16_t>(u >> 16);
    if (neg) b |= 0x8000;
    return b;
}

double weight_at(const void* w, int w_dt, int64_t j) {
    if (w_dt == 0) return bf16_to_double(static_cast<const uint16_t*>(w)[j]);
    return static_cast<double>(static_cast<const float*>(w)[j]);
}

int clamp_threads(int nthreads, int64_t work) {
    int n = nthreads > 0 ? nthreads : static_cast<int>(std::thread::hardware_concurrency());
    if (n < 1) n = 1;
    if (work < n) n = static_cast<int>(std::max<int64_t>(work, 1));
    return n;
}

template <class F>
void parallel_ranges(int64_t n, int nthreads, F fn) {
    const int nt = clamp_threads(nthreads, n);
    if (nt == 1) { fn(int64_t(0), n); return; }
    std::vector<std::thread> pool;
    for (int t = 0; t < nt; ++t) {
        const int64_t a = n * t / nt, b = n * (t + 1) / nt;
        pool.emplace_back([=] { fn(a, b); });
    }
    for (auto& th : pool) th.join();
}

// ---- one row of the forward, FP64 ---------------------------------------------------

// rstd = 1 / sqrt(mean(x^2) + eps); y = x * rstd * w (unrounded).
double row_forward(int64_t H, const double* x, const double* w, double eps, double* y) {
    double ss = 0.0;
    for (int64_t j = 0; j < H; ++j) ss += x[j] * x[j];
    const double ms = ss / static_cast<double>(H);
    const double rstd = 1.0 / std::sqrt(ms + eps);
    if (y)
        for (int64_t j = 0; j < H; ++j) y[j] = x[j] * rstd * w[j];
    return rstd;
}

// ---- one row of the backward, FP64 ---------------------------------------------------

// dx_j = rstd (g_j - xh_j c), xh = x rstd, g = dy w, c = (1/H) sum g xh; plus dh_j if given.
void row_backward(int64_t H, const double* x, const double* w, double rstd, const double* dy,
                  const double* dh, double* dx) {
    double dot = 0.0;
    for (int64_t j = 0; j < H; ++j) dot += (dy[j] * w[j]) * (x[j] * rstd);
    const double c = dot / static_cast<double>(H);
    for (int64_t j = 0; j < H; ++j) {
        const double xh = x[j] * rstd;
        const double g = dy[j] * w[j];
        double v = rstd * (g - xh * c);
        if (dh) v += dh[j];
        dx[j] = v;
    }
}

// dw_j = sum_r dy_rj x_rj rstd_r, every column in increasing row order.
// Callers pass an element accessor so the same loop serves double and BF16 inputs.
template <class GetX, class GetDy>
void columns_dw(int64_t R, int64_t H, GetX getx, GetDy getdy, const double* rstd, double* dw,
                int nthreads) {
    parallel_ranges(H, nthreads, [&](int64_t j0, int64_t j1) {
        std::vector<double> acc(static_cast<size_t>(j1 - j0), 0.0);
        for (int64_t r = 0; r < R; ++r)
            for (int64_t j = j0; j < j1; ++j)
                acc[j - j0] += getdy(r, j) * getx(r, j) * rstd[r];
        for (int64_t j = j0; j < j1; ++j) dw[j] = acc[j - j0];
    });
}

}  // namespace

extern "C" {

// ---- conversions ------------------------------------------------------------------

void oracle_bf16_from_f64(int64_t n, const double* v, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = double_to_bf16(v[i]);
}

void oracle_f64_from_bf16(int64_t n, const uint16_t* b, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = bf16_to_double(b[i]);
}

// ---- FP64 definitions on dense double arrays (used for derivative checks) ----------

// x, y: [R, H] row-major; w: [H]; rstd: [R]. y may be null.
void oracle_fwd_f64(int64_t R, int64_t H, const double* x, const double* w, double eps,
                    double* y, double* rstd, int nthreads) {
    parallel_ranges(R, nthreads, [&](int64_t a, int64_t b) {
        for (int64_t r = a; r < b; ++r)
            rstd[r] = row_forward(H, x + r * H, w, eps, y ? y + r * H : nullptr);
    });
}

// dx: [R, H]; dw: [H]; dh may be null (plain form).
void oracle_bwd_f64(int64_t R, int64_t H, const double* x, const double* w, const double* rstd,
                    const double* dy, const double* dh, double* dx, double* dw, int nthreads) {
    parallel_ranges(R, nthreads, [&](int64_t a, int64_t b) {
        for (int64_t r = a; r < b; ++r)
            row_backward(H, x + r * H, w, rstd[r], dy + r * H, dh ? dh + r * H : nullptr,
                         dx + r * H);
    });
    columns_dw(
        R, H, [&](int64_t r, int64_t j) { return x[r * H + j]; },
        [&](int64_t r, int64_t j) { return dy[r * H + j]; }, rstd, dw, nthreads);
}

// ---- the API-level oracle on BF16 bits ------------------------------------------------
// All row tensors are dense [R, H] BF16 bit arrays (the caller gathers strided views).
// w_dt: 0 = BF16 bits, 1 = FP32.  eps is the FP32 value the API receives.

// Forward; res may be null (plain form).  With res, h_out receives BF16(x + res) and
// the norm runs on it.  rstd64 may be null; when given it receives the unrounded rstd.
void oracle_train_fwd(int64_t R, int64_t H, const uint16_t* x, const uint16_t* res,
                      const void* w, int w_dt, float eps, uint16_t* h_out, uint16_t* y,
                      float* rstd, double* rstd64, int nthreads) {
    std::vector<double> wd(static_cast<size_t>(H));
    for (int64_t j = 0; j < H; ++j) wd[j] = weight_at(w, w_dt, j);
    parallel_ranges(R, nthreads, [&](int64_t a, int64_t b) {
        std::vector<double> xr(static_cast<size_t>(H)), yr(static_cast<size_t>(H));
        for (int64_t r = a; r < b; ++r) {
            for (int64_t j = 0; j < H; ++j) {
                double v = bf16_to_double(x[r * H + j]);
                if (res) {
                    // exact in double (both are BF16), then one rounding to BF16
                    const uint16_t hb = double_to_bf16(v + bf16_to_double(res[r * H + j]));
                    h_out[r * H + j] = hb;
                    v = bf16_to_double(hb);
                }
                xr[j] = v;
            }
            const double rs = row_forward(H, xr.data(), wd.data(), static_cast<double>(eps),
                                          yr.data());
            for (int64_t j = 0; j < H; ++j) y[r * H + j] = double_to_bf16(yr[j]);
            rstd[r] = static_cast<float>(rs);
            if (rstd64) rstd64[r] = rs;
        }
    });
}

// Backward with the caller's FP32 rstd.  x is the forward's normalised input (h in the
// residual form); dh may be null (plain form).  dx receives BF16 dx (grad_h with dh);
// dw64 receives the FP64 column sums.
void oracle_train_bwd(int64_t R, int64_t H, const uint16_t* x, const void* w, int w_dt,
                      const float* rstd, const uint16_t* dy, const uint16_t* dh, uint16_t* dx,
                      double* dw64, int nthreads) {
    std::vector<double> wd(static_cast<size_t>(H));
    for (int64_t j = 0; j < H; ++j) wd[j] = weight_at(w, w_dt, j);
    std::vector<double> rs(static_cast<size_t>(R));
    for (int64_t r = 0; r < R; ++r) rs[r] = static_cast<double>(rstd[r]);
    if (dx) {
        parallel_ranges(R, nthreads, [&](int64_t a, int64_t b) {
            std::vector<double> xr(static_cast<size_t>(H)), dyr(static_cast<size_t>(H)),
                dhr(static_cast<size_t>(H)), out(static_cast<size_t>(H));
            for (int64_t r = a; r < b; ++r) {
                for (int64_t j = 0; j < H; ++j) {
                    xr[j] = bf16_to_double(x[r * H + j]);
                    dyr[j] = bf16_to_double(dy[r * H + j]);
                    if (dh) dhr[j] = bf16_to_double(dh[r * H + j]);
                }
                row_backward(H, xr.data(), wd.data(), rs[r], dyr.data(),
                             dh ? dhr.data() : nullptr, out.data());
                for (int64_t j = 0; j < H; ++j) dx[r * H + j] = double_to_bf16(out[j]);
            }
        });
    }
    if (dw64) {
        columns_dw(
            R, H, [&](int64_t r, int64_t j) { return bf16_to_double(x[r * H + j]); },
            [&](int64_t r, int64_t j) { return bf16_to_double(dy[r * H + j]); }, rs.data(),
            dw64, nthreads);
    }
}

int oracle_hardware_threads(void) {
    return static_cast<int>(std::thread::hardware_concurrency());
}

}  // extern "C"
