// Training RMSNorm forward (plain and residual form) for sm_100a.
//
//   rstd_r = 1 / sqrt(mean_j x_rj^2 + eps),   y_rj = BF16(x_rj * rstd_r * w_j)
//   residual form: h_rj = BF16(x_rj + res_rj), h is stored and the norm runs on h.
// (flashinfer PR #8848 introduction and "Workload"; PR #8512 "Residual rows".)
//
// Design: one warp owns ROWS rows at a time and holds them whole in registers
// (VPT 16-byte vectors per lane per row), so every element is read from HBM once
// and the row sum of squares is a warp-shuffle tree with no shared memory or
// barrier.  The grid is persistent (SM count x resident CTAs) and walks row groups
// in order, which keeps neighbouring warps on neighbouring DRAM pages.  All row
// loads of a group are issued before any use, which keeps VPT*ROWS*16 bytes per lane
// in flight.  Squares of BF16 values are exact in FP32; each 16-byte vector is summed
// as a small tree, lanes sequentially over their vectors, then a 5-level shuffle tree.
#include "common.cuh"

namespace rmsk {

constexpr int kFwdThreads = 256;

template <int VPT, int ROWS, bool RES, bool W32>
__global__ void __launch_bounds__(kFwdThreads) fwd_kernel(const FwdParams p) {
    const int lane = threadIdx.x & 31;
    const int gwarp = (int)((blockIdx.x * kFwdThreads + threadIdx.x) >> 5);
    const int nwarps = (int)((gridDim.x * kFwdThreads) >> 5);
    const int ngroups = (p.R + ROWS - 1) / ROWS;
    const float Hf = (float)p.H;

    for (int g = gwarp; g < ngroups; g += nwarps) {
        const int r0 = g * ROWS;
        uint4 xv[ROWS][VPT];
        int64_t oy[ROWS];
#pragma unroll
        for (int q = 0; q < ROWS; ++q) {
            const int r = r0 + q;
            const bool rv = r < p.R;
            const int64_t ox = rv ? row_offset(r, p.heads, p.x.st, p.x.sk) : 0;
            oy[q] = rv ? row_offset(r, p.heads, p.y.st, p.y.sk) : 0;
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                const int v = lane + 32 * i;
                xv[q][i] = (rv && v < p.nvec) ? ld_stream16(p.x.ptr + ox + 8 * v)
                                              : make_uint4(0u, 0u, 0u, 0u);
            }
        }
        if constexpr (RES) {
            uint4 rv4[ROWS][VPT];
#pragma unroll
            for (int q = 0; q < ROWS; ++q) {
                const int r = r0 + q;
                const bool rv = r < p.R;
                const int64_t orr = rv ? row_offset(r, p.heads, p.res.st, p.res.sk) : 0;
#pragma unroll
                for (int i = 0; i < VPT; ++i) {
                    const int v = lane + 32 * i;
                    rv4[q][i] = (rv && v < p.nvec) ? ld_stream16(p.res.ptr + orr + 8 * v)
                                                   : make_uint4(0u, 0u, 0u, 0u);
                }
            }
#pragma unroll
            for (int q = 0; q < ROWS; ++q) {
                const int r = r0 + q;
                const bool rv = r < p.R;
                const int64_t oh = rv ? row_offset(r, p.heads, p.h.st, p.h.sk) : 0;
#pragma unroll
                for (int i = 0; i < VPT; ++i) {
                    float a[8], b[8];
                    unpack8(xv[q][i], a);
                    unpack8(rv4[q][i], b);
#pragma unroll
                    for (int e = 0; e < 8; ++e) a[e] = __fadd_rn(a[e], b[e]);
                    xv[q][i] = pack8(a);  // h = BF16(x + res): the norm runs on rounded h
                    const int v = lane + 32 * i;
                    if (rv && v < p.nvec) st16(p.h.ptr + oh + 8 * v, xv[q][i]);
                }
            }
        }
        float rs[ROWS];
#pragma unroll
        for (int q = 0; q < ROWS; ++q) {
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                float f[8];
                unpack8(xv[q][i], f);
                const float s01 = __fadd_rn(__fmul_rn(f[0], f[0]), __fmul_rn(f[1], f[1]));
                const float s23 = __fadd_rn(__fmul_rn(f[2], f[2]), __fmul_rn(f[3], f[3]));
                const float s45 = __fadd_rn(__fmul_rn(f[4], f[4]), __fmul_rn(f[5], f[5]));
                const float s67 = __fadd_rn(__fmul_rn(f[6], f[6]), __fmul_rn(f[7], f[7]));
                acc = __fadd_rn(acc, __fadd_rn(__fadd_rn(s01, s23), __fadd_rn(s45, s67)));
            }
            const float ss = warp_sum(acc);
            const float ms = __fdiv_rn(ss, Hf);
            rs[q] = __frcp_rn(__fsqrt_rn(__fadd_rn(ms, p.eps)));
        }
#pragma unroll
        for (int q = 0; q < ROWS; ++q) {
            if (r0 + q >= p.R) continue;
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                const int v = lane + 32 * i;
                if (v < p.nvec) {
                    float f[8], wf[8];
                    unpack8(xv[q][i], f);
                    load_w8<W32>(p.w, 8 * v, wf);
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] = __fmul_rn(__fmul_rn(f[e], rs[q]), wf[e]);
                    st16(p.y.ptr + oy[q] + 8 * v, pack8(f));
                }
            }
        }
        // lane q stores row q's rstd: one coalesced store per group
        float mine = rs[0];
#pragma unroll
        for (int q = 1; q < ROWS; ++q)
            if (lane == q) mine = rs[q];
        if (lane < ROWS && r0 + lane < p.R) p.rstd[r0 + lane] = mine;
    }
}

namespace {

template <int VPT, int ROWS, bool RES, bool W32>
cudaError_t launch_one(const FwdParams& p, cudaStream_t s) {
    auto kern = fwd_kernel<VPT, ROWS, RES, W32>;
    static int occ = -1;  // resident CTAs per SM for this instantiation
    if (occ < 0) {
        int o = 0;
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, kern, kFwdThreads, 0);
        if (e != cudaSuccess) return e;
        occ = o > 0 ? o : 1;
    }
    const int warps_per_cta = kFwdThreads / 32;
    const int64_t groups = ((int64_t)p.R + ROWS - 1) / ROWS;
    const int64_t need = (groups + warps_per_cta - 1) / warps_per_cta;
    const int64_t cap = (int64_t)device_sm_count() * occ;
    const int grid = (int)(need < cap ? need : cap);
    if (grid <= 0) return cudaSuccess;
    kern<<<grid, kFwdThreads, 0, s>>>(p);
    return cudaGetLastError();
}

template <int VPT, int ROWS_BIG>
cudaError_t launch_vpt(const FwdParams& p, bool res, bool w32, cudaStream_t s) {
    // Several rows per warp only when there are enough rows to fill the GPU with them.
    const bool big = ROWS_BIG > 1 &&
                     (int64_t)p.R >= (int64_t)device_sm_count() * 64 * ROWS_BIG * 2;
    if (big) {
        if (res) return w32 ? launch_one<VPT, ROWS_BIG, true, true>(p, s)
                            : launch_one<VPT, ROWS_BIG, true, false>(p, s);
        return w32 ? launch_one<VPT, ROWS_BIG, false, true>(p, s)
                   : launch_one<VPT, ROWS_BIG, false, false>(p, s);
    }
    if (res) return w32 ? launch_one<VPT, 1, true, true>(p, s)
                        : launch_one<VPT, 1, true, false>(p, s);
    return w32 ? launch_one<VPT, 1, false, true>(p, s) : launch_one<VPT, 1, false, false>(p, s);
}

}  // namespace

cudaError_t launch_fwd(const FwdParams& p, bool res, bool w32, cudaStream_t s) {
    if (p.R <= 0) return cudaSuccess;
    const int need = (p.nvec + 31) / 32;  // vectors per lane
    if (need <= 1) return launch_vpt<1, 4>(p, res, w32, s);
    if (need <= 2) return launch_vpt<2, 2>(p, res, w32, s);
    if (need <= 3) return launch_vpt<3, 1>(p, res, w32, s);
    if (need <= 4) return launch_vpt<4, 1>(p, res, w32, s);
    if (need <= 6) return launch_vpt<6, 1>(p, res, w32, s);
    if (need <= 8) return launch_vpt<8, 1>(p, res, w32, s);
    if (need <= 12) return launch_vpt<12, 1>(p, res, w32, s);
    if (need <= 16) return launch_vpt<16, 1>(p, res, w32, s);
    if (need <= 20) return launch_vpt<20, 1>(p, res, w32, s);
    if (need <= 24) return launch_vpt<24, 1>(p, res, w32, s);
    if (need <= 28) return launch_vpt<28, 1>(p, res, w32, s);
    return launch_vpt<32, 1>(p, res, w32, s);
}

}  // namespace rmsk
