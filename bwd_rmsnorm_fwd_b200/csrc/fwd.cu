// Training RMSNorm forward (plain and residual form) for sm_100a.
//
//   rstd_r = 1 / sqrt(mean_j x_rj^2 + eps),   y_rj = BF16(x_rj * rstd_r * w_j)
//   residual form: h_rj = BF16(x_rj + res_rj), h is stored and the norm runs on h.
// (flashinfer PR #8848 introduction and "Workload"; PR #8512 "Residual rows".)
//
// Design: every row is read from HBM once, reduced, scaled and written back once, so what
// sets the forward's speed is how many bytes are in flight per SM and how little work sits
// between a row's last load and its first store.  Many small resident CTAs with
// all of a row's loads issued before any use beat a shared-memory pipeline with one CTA
// per SM at every width and row count measured (H 256..8192, rows 1..393216), because the
// pipeline's per-row reduction, barrier and wait latencies stay exposed with few warps.
//
//   * rows of at most 4 vectors (16 bytes) per lane, H <= 1024: one warp per row (or per
//     group of ROWS rows for the narrowest widths once there are rows enough to fill the
//     GPU), a 5-level shuffle tree per row; for mid-sized row counts at H <= 256 the rows
//     pass through a 4-row per-warp cp.async ring in shared memory;
//   * wider rows: one CTA per row, every thread VPT vectors of it (2 up to H 4096, 4
//     above), warp sums met in shared memory; in the residual form at H > 4096 and many
//     rows, the rows pass through a two-row per-thread cp.async ring in shared memory.
//
// Both grids are persistent (SM count x resident CTAs) and walk rows in order, which keeps
// neighbouring CTAs on neighbouring DRAM pages.  Squares of BF16 values are exact in FP32;
// each 16-byte vector is summed as a small tree, a thread sums its vectors in order, then a
// shuffle tree (and, across warps, a sum in warp order).  rstd = rsqrtf(sum * (1/H) + eps)
// in FP32: CUDA documents rsqrtf to within 2 ulp and the FMA rounds the mean once, so rstd
// is within a few FP32 ulps of the exact value.  The forward has no barrier waits: the rings
// wait only for a thread's own copies to land.
#include "common.cuh"

namespace rmsk {

constexpr int kFwdWarpThreads = 256;

// Sum of squares of one 16-byte vector of BF16 values (exact squares, a 3-level tree).
__device__ __forceinline__ float sumsq8(const uint4& v) {
    float f[8];
    unpack8(v, f);
    const float s01 = __fadd_rn(__fmul_rn(f[0], f[0]), __fmul_rn(f[1], f[1]));
    const float s23 = __fadd_rn(__fmul_rn(f[2], f[2]), __fmul_rn(f[3], f[3]));
    const float s45 = __fadd_rn(__fmul_rn(f[4], f[4]), __fmul_rn(f[5], f[5]));
    const float s67 = __fadd_rn(__fmul_rn(f[6], f[6]), __fmul_rn(f[7], f[7]));
    return __fadd_rn(__fadd_rn(s01, s23), __fadd_rn(s45, s67));
}

// h = BF16(x + res) for one vector; the norm then runs on the rounded h.
__device__ __forceinline__ uint4 add_round8(const uint4& x, const uint4& r) {
    float a[8], b[8];
    unpack8(x, a);
    unpack8(r, b);
#pragma unroll
    for (int e = 0; e < 8; ++e) a[e] = __fadd_rn(a[e], b[e]);
    return pack8(a);
}

// y = BF16((x * rstd) * w) for one vector of columns 8v .. 8v+7.
template <bool W32>
__device__ __forceinline__ uint4 scale8(const uint4& x, float rstd, const void* w, int v) {
    float f[8], wf[8];
    unpack8(x, f);
    load_w8<W32>(w, 8 * v, wf);
#pragma unroll
    for (int e = 0; e < 8; ++e) f[e] = __fmul_rn(__fmul_rn(f[e], rstd), wf[e]);
    return pack8(f);
}

// ---- rows of <= 4 vectors per lane: one warp per row (group) -----------------------------------
// MINB: CTAs per SM the registers are capped for (launch bounds).
template <int VPT, int ROWS, bool RES, bool W32, int MINB>
__global__ void __launch_bounds__(kFwdWarpThreads, MINB) fwd_warp_kernel(const FwdParams p) {
    const int lane = threadIdx.x & 31;
    const int gwarp = (int)((blockIdx.x * kFwdWarpThreads + threadIdx.x) >> 5);
    const int nwarps = (int)((gridDim.x * kFwdWarpThreads) >> 5);
    const int ngroups = (p.R + ROWS - 1) / ROWS;
    const float invH = 1.0f / (float)p.H;

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
                    xv[q][i] = add_round8(xv[q][i], rv4[q][i]);
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
            for (int i = 0; i < VPT; ++i) acc = __fadd_rn(acc, sumsq8(xv[q][i]));
            rs[q] = rsqrtf(__fmaf_rn(warp_sum(acc), invH, p.eps));
        }
#pragma unroll
        for (int q = 0; q < ROWS; ++q) {
            if (r0 + q >= p.R) continue;
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                const int v = lane + 32 * i;
                if (v < p.nvec) st16(p.y.ptr + oy[q] + 8 * v, scale8<W32>(xv[q][i], rs[q], p.w, v));
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

// ---- narrow rows at many rows: one warp per row, a per-warp cp.async ring ------------------------
// Lane l owns vector l (and l + 32, ...) of every row; rows are taken grid-stride over the warps
// of the grid.  Each warp runs an S-row ring in shared memory filled by per-lane cp.async, so S-1
// rows of loads stay in flight per warp at no register cost; a lane reads back only what it copied
// itself and waits for its own copies only.
template <int VPT, int S, bool RES, bool W32>
__global__ void __launch_bounds__(kFwdWarpThreads) fwd_warp_ring_kernel(const FwdParams p) {
    constexpr int NTEN = RES ? 2 : 1;
    constexpr int SB = NTEN * VPT * 512;  // one row of one warp: tensors x vectors x 32 lanes x 16 B
    extern __shared__ __align__(16) unsigned char fsm[];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int nw = (int)(blockDim.x >> 5);
    const float invH = 1.0f / (float)p.H;
    unsigned char* ring = fsm + (size_t)warp * S * SB;
    const uint32_t ring_s = smem_addr(ring);
    const int gw = blockIdx.x * nw + warp;
    const int nwt = gridDim.x * nw;
    const int total = p.R > gw ? (p.R - 1 - gw) / nwt + 1 : 0;
    auto issue = [&](int j) {
        if (j < total) {
            const int r = gw + j * nwt;
            const uint32_t st = ring_s + (uint32_t)((j % S) * SB);
            const int64_t ox = row_offset(r, p.heads, p.x.st, p.x.sk);
            const int64_t orr = RES ? row_offset(r, p.heads, p.res.st, p.res.sk) : 0;
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                const int v = lane + 32 * i;
                if (v < p.nvec) {
                    cp_async16(st + (uint32_t)(i * 512 + lane * 16), p.x.ptr + ox + 8 * v);
                    if constexpr (RES)
                        cp_async16(st + (uint32_t)((VPT + i) * 512 + lane * 16), p.res.ptr + orr + 8 * v);
                }
            }
        }
        cp_async_commit();  // one group per row, empty or not: wait_group counts them
    };
#pragma unroll
    for (int j = 0; j < S - 1; ++j) issue(j);
    for (int j = 0; j < total; ++j) {
        cp_async_wait<S - 2>();  // this lane's copies of row j have landed
        const int r = gw + j * nwt;
        const unsigned char* st = ring + (j % S) * SB;
        uint4 xv[VPT];
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const bool in = lane + 32 * i < p.nvec;
            xv[i] = in ? *reinterpret_cast<const uint4*>(st + i * 512 + lane * 16)
                       : make_uint4(0u, 0u, 0u, 0u);
        }
        if constexpr (RES) {
            const int64_t oh = row_offset(r, p.heads, p.h.st, p.h.sk);
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                const int v = lane + 32 * i;
                if (v < p.nvec) {
                    xv[i] = add_round8(xv[i], *reinterpret_cast<const uint4*>(st + (VPT + i) * 512 + lane * 16));
                    st16(p.h.ptr + oh + 8 * v, xv[i]);
                }
            }
        }
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < VPT; ++i) acc = __fadd_rn(acc, sumsq8(xv[i]));
        const float rs = rsqrtf(__fmaf_rn(warp_sum(acc), invH, p.eps));
        const int64_t oy = row_offset(r, p.heads, p.y.st, p.y.sk);
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = lane + 32 * i;
            if (v < p.nvec) st16(p.y.ptr + oy + 8 * v, scale8<W32>(xv[i], rs, p.w, v));
        }
        if (lane == 0) p.rstd[r] = rs;
        issue(j + S - 1);
    }
    cp_async_wait<0>();
}

// ---- wider rows: one CTA per row ----------------------------------------------------------------
// Thread t holds vectors t, t + NT, ... (VPT of them) of the row, so a warp's loads and stores
// are whole 512-byte runs.  The warp sums meet in shared memory and every thread adds them in
// warp order (two buffers, one barrier per row).  With D >= 2 the rows pass through a ring of D
// rows in shared memory filled by per-thread cp.async: thread t copies its own vectors of the
// CTA's next D-1 rows before it reduces and writes the current one, and reads back only what it
// copied itself, so its own cp.async.wait_group is all the synchronisation the ring needs and the
// loads stay in flight through the reduction, the barrier and the stores at no register cost.
// D == 0 loads each row straight into registers.
constexpr int kFwdRowMaxThreads = 256;

template <int VPT, bool RES>
__device__ __forceinline__ void load_row(const FwdParams& p, int r, uint4 (&xv)[VPT],
                                         uint4 (&rv)[RES ? VPT : 1]) {
    const int nt = (int)blockDim.x;
    const int t = (int)threadIdx.x;
    const int64_t ox = row_offset(r, p.heads, p.x.st, p.x.sk);
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int v = t + nt * i;
        xv[i] = v < p.nvec ? ld_stream16(p.x.ptr + ox + 8 * v) : make_uint4(0u, 0u, 0u, 0u);
    }
    if constexpr (RES) {
        const int64_t orr = row_offset(r, p.heads, p.res.st, p.res.sk);
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = t + nt * i;
            rv[i] = v < p.nvec ? ld_stream16(p.res.ptr + orr + 8 * v) : make_uint4(0u, 0u, 0u, 0u);
        }
    }
}

template <int VPT, int D, bool RES, bool W32, bool PF>
__global__ void __launch_bounds__(kFwdRowMaxThreads) fwd_row_cta_kernel(const FwdParams p) {
    constexpr int NTEN = RES ? 2 : 1;
    __shared__ float red[2][kFwdRowMaxThreads / 32];
    extern __shared__ __align__(16) uint4 ring[];  // [D][NTEN][VPT][NT] 16-byte vectors
    const int nt = (int)blockDim.x;
    const int nw = nt >> 5;
    const int t = (int)threadIdx.x;
    const float invH = 1.0f / (float)p.H;
    const int G = (int)gridDim.x;
    auto slot = [&](int k, int ten, int i) -> uint4* {
        return ring + (((k % (D > 0 ? D : 1)) * NTEN + ten) * VPT + i) * nt + t;
    };
    // D >= 2: copies of the k-th row of this CTA (row blockIdx.x + k*G), one group per row
    auto issue = [&](int k) {
        const int r = (int)blockIdx.x + k * G;
        if (r < p.R) {
            const int64_t ox = row_offset(r, p.heads, p.x.st, p.x.sk);
            const int64_t orr = RES ? row_offset(r, p.heads, p.res.st, p.res.sk) : 0;
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                const int v = t + nt * i;
                if (v < p.nvec) {
                    cp_async16(smem_addr(slot(k, 0, i)), p.x.ptr + ox + 8 * v);
                    if constexpr (RES) cp_async16(smem_addr(slot(k, 1, i)), p.res.ptr + orr + 8 * v);
                }
            }
        }
        cp_async_commit();
    };
    if constexpr (D >= 2) {
#pragma unroll
        for (int k = 0; k < D - 1; ++k) issue(k);
    }
    int buf = 0;
    const uint32_t row_bytes = (uint32_t)p.nvec * 16u;
    for (int k = 0, r = blockIdx.x; r < p.R; ++k, r += G, buf ^= 1) {
        uint4 xv[VPT], rv[RES ? VPT : 1];
        if (PF && t == 0) {
            // warm L2 with this CTA's next rows (the first time all p.prefetch of them, then
            // the one that has come into range), one bulk prefetch per row and tensor
            for (int a = k == 0 ? 1 : p.prefetch; a <= p.prefetch; ++a) {
                const int rn = r + a * G;
                if (rn >= p.R) break;
                prefetch_l2(p.x.ptr + row_offset(rn, p.heads, p.x.st, p.x.sk), row_bytes);
                if constexpr (RES)
                    prefetch_l2(p.res.ptr + row_offset(rn, p.heads, p.res.st, p.res.sk), row_bytes);
            }
        }
        if constexpr (D >= 2) {
            issue(k + D - 1);
            cp_async_wait<D - 1>();  // this thread's copies of row k have landed
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                const bool in = t + nt * i < p.nvec;
                xv[i] = in ? *slot(k, 0, i) : make_uint4(0u, 0u, 0u, 0u);
                if constexpr (RES) rv[i] = in ? *slot(k, 1, i) : make_uint4(0u, 0u, 0u, 0u);
            }
        } else {
            load_row<VPT, RES>(p, r, xv, rv);
        }
        if constexpr (RES) {
            const int64_t oh = row_offset(r, p.heads, p.h.st, p.h.sk);
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                xv[i] = add_round8(xv[i], rv[i]);
                const int v = t + nt * i;
                if (v < p.nvec) st16(p.h.ptr + oh + 8 * v, xv[i]);
            }
        }
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < VPT; ++i) acc = __fadd_rn(acc, sumsq8(xv[i]));
        acc = warp_sum(acc);
        if ((t & 31) == 0) red[buf][t >> 5] = acc;
        __syncthreads();
        float ss = red[buf][0];
        for (int q = 1; q < nw; ++q) ss = __fadd_rn(ss, red[buf][q]);
        const float rs = rsqrtf(__fmaf_rn(ss, invH, p.eps));
        const int64_t oy = row_offset(r, p.heads, p.y.st, p.y.sk);
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = t + nt * i;
            if (v < p.nvec) st16(p.y.ptr + oy + 8 * v, scale8<W32>(xv[i], rs, p.w, v));
        }
        if (t == 0) p.rstd[r] = rs;
    }
    if constexpr (D >= 2) cp_async_wait<0>();
}

namespace {

template <int VPT, int ROWS, bool RES, bool W32, int MINB = 1>
cudaError_t launch_warp(const FwdParams& p, cudaStream_t s) {
    auto kern = fwd_warp_kernel<VPT, ROWS, RES, W32, MINB>;
    static PerDevice<1> occ;
    cudaError_t e = cudaSuccess;
    const int o = resident_ctas(occ, current_device(), 0, kern, kFwdWarpThreads, 0, &e);
    if (o < 0) return e;
    const int warps_per_cta = kFwdWarpThreads / 32;
    const int64_t groups = ((int64_t)p.R + ROWS - 1) / ROWS;
    const int64_t need = (groups + warps_per_cta - 1) / warps_per_cta;
    const int64_t cap = (int64_t)device_sm_count() * o;
    const int grid = (int)(need < cap ? need : cap);
    kern<<<grid, kFwdWarpThreads, 0, s>>>(p);
    return cudaGetLastError();
}

template <int VPT, int ROWS_BIG>
cudaError_t launch_warp_vpt(const FwdParams& p, bool res, bool w32, cudaStream_t s) {
    // Several rows per warp only when there are enough rows to fill the GPU with them.
    const bool big = ROWS_BIG > 1 &&
                     (int64_t)p.R >= (int64_t)device_sm_count() * 64 * ROWS_BIG * 2;
    if (big) {
        // four rows of one vector per warp: registers capped for four CTAs per SM (32 warps)
        // with a BF16 weight (no spill: H 256 x 1M 180 vs 183 us) and for per-head views (an
        // FP32 weight spills 16 bytes there, but [16384,24,256] runs 70.6 vs 76.5 us); plain
        // FP32-weight rows keep three CTAs (176 vs 184 us at 1M rows)
        if constexpr (VPT == 1 && ROWS_BIG == 4) {
            if (!w32 || p.heads > 1) {
                if (res) return w32 ? launch_warp<VPT, ROWS_BIG, true, true, 4>(p, s)
                                    : launch_warp<VPT, ROWS_BIG, true, false, 4>(p, s);
                return w32 ? launch_warp<VPT, ROWS_BIG, false, true, 4>(p, s)
                           : launch_warp<VPT, ROWS_BIG, false, false, 4>(p, s);
            }
        }
        if (res) return w32 ? launch_warp<VPT, ROWS_BIG, true, true>(p, s)
                            : launch_warp<VPT, ROWS_BIG, true, false>(p, s);
        return w32 ? launch_warp<VPT, ROWS_BIG, false, true>(p, s)
                   : launch_warp<VPT, ROWS_BIG, false, false>(p, s);
    }
    if (res) return w32 ? launch_warp<VPT, 1, true, true>(p, s)
                        : launch_warp<VPT, 1, true, false>(p, s);
    return w32 ? launch_warp<VPT, 1, false, true>(p, s) : launch_warp<VPT, 1, false, false>(p, s);
}

// One warp per row with an S-row cp.async ring per warp (8-warp CTAs).
template <int VPT, int S, bool RES, bool W32>
cudaError_t launch_warp_ring(const FwdParams& p, cudaStream_t s) {
    auto kern = fwd_warp_ring_kernel<VPT, S, RES, W32>;
    const size_t smem = (size_t)(kFwdWarpThreads / 32) * S * (RES ? 2 : 1) * VPT * 512;
    static SmemGrant granted;
    static PerDevice<1> occ;
    const int dev = current_device();
    cudaError_t e = cudaSuccess;
    if (smem > 48 * 1024 && (e = grant_smem(granted, dev, kern, smem)) != cudaSuccess) return e;
    const int o = resident_ctas(occ, dev, 0, kern, kFwdWarpThreads, smem, &e);
    if (o < 0) return e;
    const int64_t need = ((int64_t)p.R + kFwdWarpThreads / 32 - 1) / (kFwdWarpThreads / 32);
    const int64_t cap = (int64_t)device_sm_count() * o;
    const int grid = (int)(need < cap ? need : cap);
    kern<<<grid, kFwdWarpThreads, smem, s>>>(p);
    return cudaGetLastError();
}

// One CTA per row: ceil(nvec / (32 VPT)) warps; a D-row cp.async ring when D >= 2.  PF: the
// L2 prefetch of the CTA's next rows is compiled in (its registers would cost resident CTAs
// where it is off: 40 -> 44 registers, 12 -> 10 CTAs per SM at H 2048, FP32 weight).
template <int VPT, int D, bool RES, bool W32, bool PF = false>
cudaError_t launch_row_cta(const FwdParams& p, cudaStream_t s) {
    if constexpr (!PF && D == 0) {
        if (p.prefetch > 0) return launch_row_cta<VPT, D, RES, W32, true>(p, s);
    }
    auto kern = fwd_row_cta_kernel<VPT, D, RES, W32, PF>;
    const int warps = (p.nvec + 32 * VPT - 1) / (32 * VPT);
    if (warps * 32 > kFwdRowMaxThreads) return cudaErrorInvalidConfiguration;
    const size_t smem = D >= 2 ? (size_t)D * (RES ? 2 : 1) * VPT * warps * 32 * 16 : 0;
    const int dev = current_device();
    cudaError_t e = cudaSuccess;
    if constexpr (D >= 2) {
        // the ring of the widest row this instantiation serves (above the 48 KB default)
        static SmemGrant granted;
        const size_t most = (size_t)D * (RES ? 2 : 1) * VPT * kFwdRowMaxThreads * 16;
        if ((e = grant_smem(granted, dev, kern, most)) != cudaSuccess) return e;
    }
    static PerDevice<kFwdRowMaxThreads / 32 + 1> occ;  // by warp count
    const int o = resident_ctas(occ, dev, warps, kern, warps * 32, smem, &e);
    if (o < 0) return e;
    const int64_t cap = (int64_t)device_sm_count() * o;
    const int grid = (int)(p.R < cap ? p.R : cap);
    kern<<<grid, warps * 32, smem, s>>>(p);
    return cudaGetLastError();
}

template <int VPT, int D>
cudaError_t launch_row_cta_vpt(const FwdParams& p, bool res, bool w32, cudaStream_t s) {
    if (res) return w32 ? launch_row_cta<VPT, D, true, true>(p, s)
                        : launch_row_cta<VPT, D, true, false>(p, s);
    return w32 ? launch_row_cta<VPT, D, false, true>(p, s)
               : launch_row_cta<VPT, D, false, false>(p, s);
}

}  // namespace

constexpr int kFwdRingMinRows = 32768;
constexpr int kFwdWarpRingRows[2] = {8192, 131072};

cudaError_t launch_fwd(const FwdParams& p, bool res, bool w32, cudaStream_t s) {
    if (p.R <= 0) return cudaSuccess;
    const int need = (p.nvec + 31) / 32;  // vectors per lane of a warp-wide row
    if (need <= 1) {
        // Mid-sized plain forwards of rows of one vector per lane (H <= 256) keep more loads in
        // flight through a 4-row cp.async ring per warp (measured: [1024,24,256] 7.4 vs 8.7 us,
        // [16384,4,256] 14.4 vs 16.3 us); below the window the ring's start-up costs more than it
        // brings, above it the register kernel's four rows per warp already saturate HBM.
        if (!res && p.R >= kFwdWarpRingRows[0] && p.R < kFwdWarpRingRows[1])
            return w32 ? launch_warp_ring<1, 4, false, true>(p, s) : launch_warp_ring<1, 4, false, false>(p, s);
        return launch_warp_vpt<1, 4>(p, res, w32, s);
    }
    if (need <= 2) return launch_warp_vpt<2, 2>(p, res, w32, s);
    if (need <= 3) return launch_warp_vpt<3, 1>(p, res, w32, s);
    if (need <= 4) return launch_warp_vpt<4, 1>(p, res, w32, s);
    // H 4096 from 32768 rows: four vectors per thread (128-thread CTAs), twice the loads in
    // flight per thread (measured: H 4096 x 131072 FP32 w 335 vs 356 us, BF16 w 344 vs 347 us,
    // residual x 65537 335 vs 350 us; 3-5 % slower at 16384 rows, mixed at H 3072)
    if (p.nvec <= 384 || (p.nvec <= 512 && p.R < kFwdRingMinRows))
        return launch_row_cta_vpt<2, 0>(p, res, w32, s);
    // The residual form reads two rows per row: there a two-row cp.async ring keeps enough
    // bytes in flight to pay for itself once every CTA walks many rows (measured: H 6144 x
    // 65537 rows 513 vs 529 us); for one input row it costs more than it brings.
    if (res && p.R >= kFwdRingMinRows)
        return w32 ? launch_row_cta<4, 2, true, true>(p, s) : launch_row_cta<4, 2, true, false>(p, s);
    return launch_row_cta_vpt<4, 0>(p, res, w32, s);
}

}  // namespace rmsk
