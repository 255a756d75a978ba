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
// rstd = rsqrtf(sum * (1/H) + eps) in FP32: CUDA documents rsqrtf to within 2 ulp, and
// the FMA rounds the mean once, so rstd is within a few FP32 ulps of the exact value.
#include "common.cuh"

namespace rmsk {

constexpr int kFwdThreads = 256;

__device__ __forceinline__ void named_bar(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

template <int VPT, int ROWS, bool RES, bool W32>
__global__ void __launch_bounds__(kFwdThreads) fwd_kernel(const FwdParams p) {
    const int lane = threadIdx.x & 31;
    const int gwarp = (int)((blockIdx.x * kFwdThreads + threadIdx.x) >> 5);
    const int nwarps = (int)((gridDim.x * kFwdThreads) >> 5);
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
            rs[q] = rsqrtf(__fmaf_rn(ss, invH, p.eps));
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

// ---- few wide rows: one CTA per row -----------------------------------------------------------
// Below a pipeline's worth of rows per SM, a row wider than 4 vectors per lane is spread over
// the warps of one CTA (thread t holds vectors t, t + NT, ...; at most 4 of them), so R rows
// occupy R SMs instead of R/8, and the code stays short: after an L2 flush its first fetch is
// part of the call's latency.  The warp sums meet in shared memory and every thread adds them
// in warp order (two buffers, one barrier per row).
constexpr int kFwdRowMaxThreads = 256;

template <int VPT, bool RES, bool W32>
__global__ void __launch_bounds__(kFwdRowMaxThreads) fwd_row_cta_kernel(const FwdParams p) {
    __shared__ float red[2][kFwdRowMaxThreads / 32];
    const int nt = (int)blockDim.x;
    const int nw = nt >> 5;
    const int t = (int)threadIdx.x;
    const float invH = 1.0f / (float)p.H;
    int buf = 0;
    for (int r = blockIdx.x; r < p.R; r += gridDim.x, buf ^= 1) {
        const int64_t ox = row_offset(r, p.heads, p.x.st, p.x.sk);
        uint4 xv[VPT];
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = t + nt * i;
            xv[i] = v < p.nvec ? ld_stream16(p.x.ptr + ox + 8 * v) : make_uint4(0u, 0u, 0u, 0u);
        }
        if constexpr (RES) {
            const int64_t orr = row_offset(r, p.heads, p.res.st, p.res.sk);
            const int64_t oh = row_offset(r, p.heads, p.h.st, p.h.sk);
            uint4 rv4[VPT];
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                const int v = t + nt * i;
                rv4[i] = v < p.nvec ? ld_stream16(p.res.ptr + orr + 8 * v)
                                    : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                float a[8], b[8];
                unpack8(xv[i], a);
                unpack8(rv4[i], b);
#pragma unroll
                for (int e = 0; e < 8; ++e) a[e] = __fadd_rn(a[e], b[e]);
                xv[i] = pack8(a);  // h = BF16(x + res): the norm runs on rounded h
                const int v = t + nt * i;
                if (v < p.nvec) st16(p.h.ptr + oh + 8 * v, xv[i]);
            }
        }
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            float f[8];
            unpack8(xv[i], f);
            const float s01 = __fadd_rn(__fmul_rn(f[0], f[0]), __fmul_rn(f[1], f[1]));
            const float s23 = __fadd_rn(__fmul_rn(f[2], f[2]), __fmul_rn(f[3], f[3]));
            const float s45 = __fadd_rn(__fmul_rn(f[4], f[4]), __fmul_rn(f[5], f[5]));
            const float s67 = __fadd_rn(__fmul_rn(f[6], f[6]), __fmul_rn(f[7], f[7]));
            acc = __fadd_rn(acc, __fadd_rn(__fadd_rn(s01, s23), __fadd_rn(s45, s67)));
        }
        acc = warp_sum(acc);
        if ((t & 31) == 0) red[buf][t >> 5] = acc;
        __syncthreads();
        float ss = red[buf][0];
        for (int k = 1; k < nw; ++k) ss = __fadd_rn(ss, red[buf][k]);
        const float rs = rsqrtf(__fmaf_rn(ss, invH, p.eps));
        const int64_t oy = row_offset(r, p.heads, p.y.st, p.y.sk);
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = t + nt * i;
            if (v < p.nvec) {
                float f[8], wf[8];
                unpack8(xv[i], f);
                load_w8<W32>(p.w, 8 * v, wf);
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = __fmul_rn(__fmul_rn(f[e], rs), wf[e]);
                st16(p.y.ptr + oy + 8 * v, pack8(f));
            }
        }
        if (t == 0) p.rstd[r] = rs;
    }
}

// ---- wide rows: bulk-copy pipeline ------------------------------------------------------------
// Warp 0 streams P rows per slot (x, and the residual in the residual form) into a ring of
// shared-memory stages with cp.async.bulk; L slots of ST consumer threads each own one row
// at a time: sum of squares (packed FP32 pairs), a shuffle tree plus a named barrier over
// the slot's warps, then y = (x * rstd) * w stored straight to global memory.  The CTA
// takes a contiguous row range split evenly between its slots.  Waits are bounded; a wait
// that gives up sets the status word and the pipeline stops waiting (see the backward).

// status word of the forward kernels (they take no workspace); read by rms_status(NULL, .)
__device__ unsigned g_fwd_status;

constexpr int kFwdMaxStages = 16;
constexpr int kFwdHeader = 2048;  // barriers (256 B), flags (16 B), slot reduction buffers

struct FwdStaged {
    int32_t n_stages;
    int32_t stage_bytes;
    int32_t tensor_bytes;
};

template <int ST, int VPT, int L, int P, bool RES, bool W32>
__global__ void __launch_bounds__(32 + ST * L, 1)
    fwd_staged_kernel(const FwdParams p, const FwdStaged sc, const __grid_constant__ RowMaps tm) {
    static_assert(ST >= 32 ? ST % 32 == 0 : 32 % ST == 0, "slot must tile warps");
    static_assert((ST * L) % 32 == 0, "consumers must fill whole warps");
    constexpr int SW = ST >= 32 ? ST / 32 : 1;  // warps per slot
    constexpr int NCW = ST * L / 32;
    constexpr int RT = L * P;
    constexpr int NTEN = RES ? 2 : 1;
    static_assert(16 * kFwdMaxStages + 16 + (ST > 32 ? L * 2 * P * SW * 4 : 0) <= kFwdHeader,
                  "slot reduction buffers must fit in the header");
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 16 * kFwdMaxStages);
    float* red = reinterpret_cast<float*>(smem + 16 * kFwdMaxStages + 16);  // [L][2][P][SW]
    unsigned char* stages = smem + kFwdHeader;
    const int NS = sc.n_stages;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int H = p.H;
    const int nvec = p.nvec;
    const uint32_t row_bytes = (uint32_t)H * 2u;
    const int64_t limit = p.wait_cycles;
    auto full_bar = [&](int s) { return smem_addr(&bars[s]); };
    auto empty_bar = [&](int s) { return smem_addr(&bars[kFwdMaxStages + s]); };
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), NCW);
        }
        *abort_flag = 0;
        mbar_init_fence();
    }
    __syncthreads();
    const int64_t lo = (int64_t)p.R * blockIdx.x / gridDim.x;
    const int64_t hi = (int64_t)p.R * (blockIdx.x + 1) / gridDim.x;
    auto sbase = [&](int s) { return (int)(lo + (hi - lo) * s / L); };
    int maxlen = 0;
#pragma unroll
    for (int s = 0; s < L; ++s) maxlen = max(maxlen, sbase(s + 1) - sbase(s));
    const int nt = (maxlen + P - 1) / P;

    if (warp == 0) {
        // tensor loads also need a 128-byte aligned destination (checked once, used for both
        // the byte count and the copies)
        const bool tma_ok = (smem_addr(stages) & 127u) == 0 && (row_bytes & 127u) == 0;
        int j = 0;
        for (; j < nt; ++j) {
            const int stage = j % NS;
            const uint32_t ph = (uint32_t)(j / NS) & 1u;
            if (j >= NS && !mbar_wait_bounded(empty_bar(stage), ph ^ 1u, limit)) {
                if (lane == 0) { *abort_flag = 1; atomicOr(&g_fwd_status, kStatusTimeout); }
            }
            __syncwarp();
            if (*abort_flag) break;
            uint32_t bytes = 0;  // a TMA box always lands whole (rows past the end as 0)
#pragma unroll
            for (int s = 0; s < L; ++s) {
                const int n = min(P, sbase(s + 1) - (sbase(s) + j * P));
                if (n > 0)
#pragma unroll
                    for (int ten = 0; ten < NTEN; ++ten)
                        bytes += (uint32_t)(tm.use[ten] && tma_ok ? P : n) * row_bytes;
            }
            if (lane == 0) mbar_arrive_expect_tx(full_bar(stage), bytes);
            __syncwarp();
            const uint32_t sb = smem_addr(stages + (size_t)stage * sc.stage_bytes);
            // one TMA box per (tensor, slot) for equally spaced rows of H <= 256, one bulk copy
            // per (tensor, slot) for contiguous rows, else one bulk copy per row
            for (int c = lane; c < L * NTEN; c += 32) {
                const int ten = c / L;
                const int s = c - ten * L;
                const RowsIn& src = ten == 0 ? p.x : p.res;
                const int row0 = sbase(s) + j * P;
                const int n = min(P, sbase(s + 1) - row0);
                if (n <= 0) continue;
                const uint32_t dst =
                    sb + (uint32_t)ten * sc.tensor_bytes + (uint32_t)(s * P) * row_bytes;
                if (tm.use[ten] && tma_ok)
                    tma_load_rows(dst, &tm.map[ten], row0, full_bar(stage));
                else if (rows_contiguous(src, p.heads, H))
                    bulk_load(dst, src.ptr + row_offset(row0, p.heads, src.st, src.sk),
                              (uint32_t)n * row_bytes, full_bar(stage));
            }
            for (int c = lane; c < RT * NTEN; c += 32) {
                const int ten = c / RT;
                const int rr = c - ten * RT;
                const int s = rr / P;
                const int q = rr - s * P;
                const int row = sbase(s) + j * P + q;
                const RowsIn& src = ten == 0 ? p.x : p.res;
                if (row < sbase(s + 1) && !(tm.use[ten] && tma_ok) && !rows_contiguous(src, p.heads, H)) {
                    bulk_load(sb + (uint32_t)ten * sc.tensor_bytes + (uint32_t)rr * row_bytes,
                              src.ptr + row_offset(row, p.heads, src.st, src.sk), row_bytes,
                              full_bar(stage));
                }
            }
            __syncwarp();
        }
        if (lane == 0) {
            for (int i = 0; i < NS && i < j; ++i) {
                const int jj = j - 1 - i;
                mbar_wait_bounded(full_bar(jj % NS), (uint32_t)(jj / NS) & 1u,
                                  limit > kDefaultWaitCycles ? limit : kDefaultWaitCycles);
            }
        }
        return;
    }

    const int ctid = threadIdx.x - 32;
    const int slot = ctid / ST;
    const int ts = ctid - slot * ST;
    const int wis = ts >> 5;
    const int base = sbase(slot);
    const int endr = sbase(slot + 1);
    const float invH = 1.0f / (float)H;
    float2 w2[VPT][4];
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int v = ts + ST * i;
        float wf[8];
        if (v < nvec) {
            load_w8<W32>(p.w, 8 * v, wf);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) wf[e] = 0.f;
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) w2[i][k] = make_float2(wf[2 * k], wf[2 * k + 1]);
    }
    int buf = 0;
    for (int t = 0; t < nt; ++t) {
        const int stage = t % NS;
        const uint32_t ph = (uint32_t)(t / NS) & 1u;
        if (!*abort_flag && !mbar_wait_bounded(full_bar(stage), ph, limit)) {
            *abort_flag = 1;
            if (lane == 0) atomicOr(&g_fwd_status, kStatusTimeout);
        }
        const unsigned char* sbp = stages + (size_t)stage * sc.stage_bytes;
        const uint4* sx = reinterpret_cast<const uint4*>(sbp + (size_t)(slot * P) * row_bytes);
        const uint4* sr = reinterpret_cast<const uint4*>(sbp + sc.tensor_bytes +
                                                         (size_t)(slot * P) * row_bytes);
        uint4 hv[RES ? P : 1][RES ? VPT : 1];
        float ss[P];
#pragma unroll
        for (int q = 0; q < P; ++q) {
            const int row = base + t * P + q;
            const bool ok = row < endr;
            float2 a2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                const int v = ts + ST * i;
                if (v < nvec) {
                    uint4 xr = sx[q * nvec + v];
                    if constexpr (RES) {
                        // h = BF16(x + residual); the norm runs on the rounded h
                        const uint4 rr = sr[q * nvec + v];
                        xr.x = pack2(add2(bf16x2_to_f2(xr.x), bf16x2_to_f2(rr.x)));
                        xr.y = pack2(add2(bf16x2_to_f2(xr.y), bf16x2_to_f2(rr.y)));
                        xr.z = pack2(add2(bf16x2_to_f2(xr.z), bf16x2_to_f2(rr.z)));
                        xr.w = pack2(add2(bf16x2_to_f2(xr.w), bf16x2_to_f2(rr.w)));
                        hv[q][i] = xr;
                        if (ok) st16(p.h.ptr + row_offset(row, p.heads, p.h.st, p.h.sk) + 8 * v, xr);
                    }
                    const uint32_t xw[4] = {xr.x, xr.y, xr.z, xr.w};
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float2 x2 = bf16x2_to_f2(xw[k]);
                        a2 = fma2(x2, x2, a2);  // squares of BF16 values are exact
                    }
                }
            }
            ss[q] = group_sum<(ST < 32 ? ST : 32)>(a2.x + a2.y);
        }
        if constexpr (SW > 1) {
            if (lane == 0) {
#pragma unroll
                for (int q = 0; q < P; ++q) red[((slot * 2 + buf) * P + q) * SW + wis] = ss[q];
            }
            named_bar(1 + slot, ST);
#pragma unroll
            for (int q = 0; q < P; ++q)
                ss[q] = warp_sum(lane < SW ? red[((slot * 2 + buf) * P + q) * SW + lane] : 0.f);
            buf ^= 1;
        }
#pragma unroll
        for (int q = 0; q < P; ++q) {
            const int row = base + t * P + q;
            if (row >= endr) continue;
            const float rstd = rsqrtf(__fmaf_rn(ss[q], invH, p.eps));
            const float2 rs2 = make_float2(rstd, rstd);
            uint16_t* yrow = p.y.ptr + row_offset(row, p.heads, p.y.st, p.y.sk);
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                const int v = ts + ST * i;
                if (v >= nvec) continue;
                uint4 xr;
                if constexpr (RES) xr = hv[q][i]; else xr = sx[q * nvec + v];
                const uint32_t xw[4] = {xr.x, xr.y, xr.z, xr.w};
                uint32_t out[4];
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    out[k] = pack2(mul2(mul2(bf16x2_to_f2(xw[k]), rs2), w2[i][k]));
                st16(yrow + 8 * v, make_uint4(out[0], out[1], out[2], out[3]));
            }
            if (ts == 0) p.rstd[row] = rstd;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(stage));
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

// One CTA per row, 4 vectors per thread: ceil(nvec / 128) warps (2..8 for H in (1024, 8192]).
template <bool RES, bool W32>
cudaError_t launch_row_cta(const FwdParams& p, cudaStream_t s) {
    constexpr int kVpt = 4;
    auto kern = fwd_row_cta_kernel<kVpt, RES, W32>;
    const int warps = (p.nvec + 32 * kVpt - 1) / (32 * kVpt);
    if (warps * 32 > kFwdRowMaxThreads) return cudaErrorInvalidConfiguration;
    static int occ[kFwdRowMaxThreads / 32 + 1] = {};  // resident CTAs per SM, by warp count
    if (occ[warps] == 0) {
        int o = 0;
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, kern, warps * 32, 0);
        if (e != cudaSuccess) return e;
        occ[warps] = o > 0 ? o : 1;
    }
    const int64_t cap = (int64_t)device_sm_count() * occ[warps];
    const int grid = (int)(p.R < cap ? p.R : cap);
    kern<<<grid, warps * 32, 0, s>>>(p);
    return cudaGetLastError();
}

template <int ST, int VPT, int L, int P, bool RES, bool W32>
cudaError_t launch_staged(const FwdParams& p, cudaStream_t s) {
    auto kern = fwd_staged_kernel<ST, VPT, L, P, RES, W32>;
    constexpr int NT = 32 + ST * L;
    constexpr size_t kBudget = 220 * 1024;
    FwdStaged sc;
    sc.tensor_bytes = L * P * p.H * 2;
    sc.stage_bytes = (RES ? 2 : 1) * sc.tensor_bytes;
    int ns = (int)((kBudget - kFwdHeader) / sc.stage_bytes);
    if (ns > kFwdMaxStages) ns = kFwdMaxStages;
    if (ns < 2) return cudaErrorInvalidConfiguration;
    sc.n_stages = ns;
    const size_t smem = kFwdHeader + (size_t)ns * sc.stage_bytes;
    static size_t smem_set = 0;
    if (smem > smem_set) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        smem_set = smem;
    }
    int64_t need = ((int64_t)p.R + L * 4 - 1) / (L * 4);
    const int64_t cap = device_sm_count();
    const int grid = (int)(need < cap ? need : cap);
    RowMaps tm;
    const RowsIn views[2] = {p.x, p.res};
    make_row_maps(&tm, views, RES ? 2 : 1, p.heads, p.H, p.R, P);
    kern<<<grid, NT, smem, s>>>(p, sc, tm);
    return cudaGetLastError();
}

// Rows of a slot per stage: the largest of 8, 4, 2 that leaves room for two stages (the
// larger the tile, the more rows each barrier, reduction and wait is spread over).
template <int ST, int VPT, int L, bool RES, bool W32>
cudaError_t launch_staged_p(const FwdParams& p, cudaStream_t s) {
    constexpr size_t kRoom = 220 * 1024 - kFwdHeader;
    const size_t row = (size_t)(RES ? 2 : 1) * L * p.H * 2;
    if (2 * 8 * row <= kRoom) return launch_staged<ST, VPT, L, 8, RES, W32>(p, s);
    if (2 * 4 * row <= kRoom) return launch_staged<ST, VPT, L, 4, RES, W32>(p, s);
    return launch_staged<ST, VPT, L, 2, RES, W32>(p, s);
}

template <bool RES, bool W32>
cudaError_t dispatch_staged(const FwdParams& p, cudaStream_t s) {
    // ST threads per slot (narrow rows share a warp), VPT vectors per thread, L slots
    const int nv = p.nvec;
    if (nv <= 32) return launch_staged_p<16, 2, 16, RES, W32>(p, s);
    if (nv <= 64) return launch_staged_p<32, 2, 8, RES, W32>(p, s);
    if (nv <= 128) return launch_staged_p<64, 2, 4, RES, W32>(p, s);
    if (nv <= 192) return launch_staged_p<64, 3, 4, RES, W32>(p, s);
    if (nv <= 256) return launch_staged_p<64, 4, 4, RES, W32>(p, s);
    if (nv <= 384) return launch_staged_p<128, 3, 2, RES, W32>(p, s);
    if (nv <= 512) return launch_staged_p<128, 4, 2, RES, W32>(p, s);
    if (nv <= 640) return launch_staged_p<128, 5, 2, RES, W32>(p, s);
    if (nv <= 768) return launch_staged_p<256, 3, 1, RES, W32>(p, s);
    return launch_staged_p<256, 4, 1, RES, W32>(p, s);
}

}  // namespace

// Rows below this count take the register kernel: too few rows per SM to fill a pipeline.
constexpr int kFwdStagedMinRowsPerSm = 16;

cudaError_t fwd_status_take(cudaStream_t s, unsigned* word) {
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(word, g_fwd_status, sizeof(unsigned));
    if (e != cudaSuccess || !*word) return e;
    const unsigned zero = 0;
    return cudaMemcpyToSymbol(g_fwd_status, &zero, sizeof zero);
}

cudaError_t launch_fwd(const FwdParams& p, bool res, bool w32, cudaStream_t s) {
    if (p.R <= 0) return cudaSuccess;
    if ((int64_t)p.R >= (int64_t)kFwdStagedMinRowsPerSm * device_sm_count()) {
        if (res) return w32 ? dispatch_staged<true, true>(p, s) : dispatch_staged<true, false>(p, s);
        return w32 ? dispatch_staged<false, true>(p, s) : dispatch_staged<false, false>(p, s);
    }
    const int need = (p.nvec + 31) / 32;  // vectors per lane of a warp-wide row
    if (need <= 1) return launch_vpt<1, 4>(p, res, w32, s);
    if (need <= 2) return launch_vpt<2, 2>(p, res, w32, s);
    if (need <= 3) return launch_vpt<3, 1>(p, res, w32, s);
    if (need <= 4) return launch_vpt<4, 1>(p, res, w32, s);
    if (res) return w32 ? launch_row_cta<true, true>(p, s) : launch_row_cta<true, false>(p, s);
    return w32 ? launch_row_cta<false, true>(p, s) : launch_row_cta<false, false>(p, s);
}

}  // namespace rmsk
