// Training RMSNorm backward for sm_100a: dx (BF16) and dw (FP32).
//
//   xh = x * rstd,  g = dy * w,  c_r = (1/H) sum_j g_rj xh_rj
//   dx_rj = rstd_r * (g_rj - xh_rj * c_r)        (+ dh_rj in the residual form)
//   dw_j  = sum_r dy_rj * xh_rj
// (flashinfer PR #8848 introduction; PR #8512 introduction and "Residual rows".)
//
// dw summation orders (PR #8512 introduction; PR #8848 introduction and the review
// comment on blocked FP32 accumulation):
//
// * deterministic: rows are cut into blocks of B rows.  A block is summed in row order
//   with exact products (p + e == dy * xh) and TwoSum, then becomes one FP64 value
//   (sum + compensation).  L consecutive blocks form a chunk, folded left to right in
//   FP64.  Chunk partials are cut into S contiguous segments, each folded left to
//   right, and the segment sums are folded left to right and rounded once to FP32.
//   B, L and S depend only on the row count and H, so the bits never depend on the
//   grid or on the SM count.  Three programs produce exactly these bits:
//     - bwd_small_kernel: one launch; row tasks compute dx, column tasks walk every
//       row of a 64-column strip and do the whole fold (used for small row counts);
//     - bwd_large_kernel<DET> + bwd_fold_kernel: CTAs take whole chunks (each slot of
//       the CTA one block), write FP64 chunk partials to the workspace, and the fold
//       kernel (launched with programmatic dependent launch) finishes the order.
// * non-deterministic: each CTA takes a contiguous row range; every thread sums eight
//   rows at a time in FP32 (one FMA per element), adds each eight-row block into an
//   FP64 accumulator in shared memory, and the CTA adds its totals into an FP64
//   workspace vector with atomics.  The last CTA to finish (atomic ticket) rounds the
//   vector to FP32 dw and clears it for the next call.
//
// The large kernels give each CTA L "slots" of SW warps; a slot owns one row at a time
// and every thread of the slot owns VPT 16-byte column vectors, so the dw state of a
// column stays in one thread's registers for the whole block.  The per-row dot
// product is a warp-shuffle tree plus, for multi-warp slots, a named barrier over the
// slot's warps with a double-buffered shared exchange.  P rows are loaded before any
// is used.
#include "common.cuh"

namespace rmsk {

__device__ __forceinline__ void named_bar(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ============================================================================================
// Large-row kernel: deterministic chunk partials or non-deterministic grid combine.
// ============================================================================================

template <int SW, int VPT, int L, int P, bool DET, bool RES, bool W32>
__global__ void __launch_bounds__(SW * 32 * L)
    bwd_large_kernel(const BwdParams p) {
    constexpr int ST = SW * 32;  // threads per slot
    constexpr int NT = ST * L;   // threads per CTA
    extern __shared__ __align__(16) unsigned char smem_raw[];
    double* sm64 = reinterpret_cast<double*>(smem_raw);  // [L][nvec*8]
    __shared__ float red[L][2][P][SW];

    const int tid = threadIdx.x;
    const int slot = tid / ST;
    const int ts = tid - slot * ST;
    const int wis = ts >> 5;
    const int lane = tid & 31;
    const int H = p.H;
    const int nvec = p.nvec;
    const float Hf = (float)H;
    double* my64 = sm64 + (size_t)slot * nvec * 8;

    // this thread's weights (FP32)
    float wv[VPT][8];
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int v = ts + ST * i;
        if (v < nvec) {
            load_w8<W32>(p.w, 8 * v, wv[i]);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) wv[i][e] = 0.f;
        }
    }

    float s_[VPT][8], c_[VPT][8];  // DET: TwoSum state; NONDET: s_ = eight-row block sum
    int buf = 0;

    auto zero_state = [&]() {
#pragma unroll
        for (int i = 0; i < VPT; ++i)
#pragma unroll
            for (int e = 0; e < 8; ++e) { s_[i][e] = 0.f; c_[i][e] = 0.f; }
    };

    // Process rows r .. r+P-1 of this slot (rows >= r_end are padding).
    auto do_rows = [&](int r, int r_end) {
        uint4 xv[P][VPT], dyv[P][VPT];
        uint4 dhv[RES ? P : 1][VPT];
        float rs[P];
        int64_t odx[P];
#pragma unroll
        for (int q = 0; q < P; ++q) {
            const int rr = r + q;
            const bool rv = rr < r_end;
            const int64_t ox = rv ? row_offset(rr, p.heads, p.x.st, p.x.sk) : 0;
            const int64_t ody = rv ? row_offset(rr, p.heads, p.dy.st, p.dy.sk) : 0;
            odx[q] = rv ? row_offset(rr, p.heads, p.dx.st, p.dx.sk) : 0;
            rs[q] = rv ? __ldg(p.rstd + rr) : 0.f;
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                const int v = ts + ST * i;
                const bool ok = rv && v < nvec;
                xv[q][i] = ok ? ld_stream16(p.x.ptr + ox + 8 * v) : make_uint4(0u, 0u, 0u, 0u);
                dyv[q][i] = ok ? ld_stream16(p.dy.ptr + ody + 8 * v) : make_uint4(0u, 0u, 0u, 0u);
            }
            if constexpr (RES) {
                const int64_t odh = rv ? row_offset(rr, p.heads, p.dh.st, p.dh.sk) : 0;
#pragma unroll
                for (int i = 0; i < VPT; ++i) {
                    const int v = ts + ST * i;
                    const bool ok = rv && v < nvec;
                    dhv[q][i] = ok ? ld_stream16(p.dh.ptr + odh + 8 * v)
                                   : make_uint4(0u, 0u, 0u, 0u);
                }
            }
        }
        // per-thread partial dot products sum_j g_j xh_j
        float dot[P];
#pragma unroll
        for (int q = 0; q < P; ++q) {
            float d = 0.f;
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                float xf[8], gf[8];
                unpack8(xv[q][i], xf);
                unpack8(dyv[q][i], gf);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    d = __fmaf_rn(__fmul_rn(gf[e], wv[i][e]), __fmul_rn(xf[e], rs[q]), d);
            }
            dot[q] = warp_sum(d);
        }
        if constexpr (SW > 1) {
            if (lane == 0) {
#pragma unroll
                for (int q = 0; q < P; ++q) red[slot][buf][q][wis] = dot[q];
            }
            named_bar(1 + slot, ST);
#pragma unroll
            for (int q = 0; q < P; ++q) {
                float d = 0.f;
#pragma unroll
                for (int w2 = 0; w2 < SW; ++w2) d = __fadd_rn(d, red[slot][buf][q][w2]);
                dot[q] = d;
            }
            buf ^= 1;
        }
        // dx and the dw accumulation, rows in increasing order
#pragma unroll
        for (int q = 0; q < P; ++q) {
            if (r + q >= r_end) continue;
            const float cr = __fdiv_rn(dot[q], Hf);
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                const int v = ts + ST * i;
                if (v >= nvec) continue;
                float xf[8], df[8], out[8];
                unpack8(xv[q][i], xf);
                unpack8(dyv[q][i], df);
                float hf[8];
                if constexpr (RES) unpack8(dhv[q][i], hf);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float xh = __fmul_rn(xf[e], rs[q]);
                    const float g = __fmul_rn(df[e], wv[i][e]);
                    float o = __fmul_rn(rs[q], __fmaf_rn(-xh, cr, g));
                    if constexpr (RES) o = __fadd_rn(o, hf[e]);
                    out[e] = o;
                    if constexpr (DET) {
                        twosum_product(df[e], xh, s_[i][e], c_[i][e]);
                    } else {
                        s_[i][e] = __fmaf_rn(df[e], xh, s_[i][e]);
                    }
                }
                st16(p.dx.ptr + odx[q] + 8 * v, pack8(out));
            }
        }
    };

    if constexpr (DET) {
        const int B = p.block_rows;
        const int CH = B * L;
        for (int k = blockIdx.x; k < p.n_chunks; k += gridDim.x) {
            const int row0 = k * CH + slot * B;
            const int row_end = min(row0 + B, p.R);
            zero_state();
            for (int r = row0; r < row_end; r += P) do_rows(r, row_end);
            const int nb = min(L, (p.R - k * CH + B - 1) / B);  // non-empty blocks of chunk k
            if constexpr (L == 1) {
#pragma unroll
                for (int i = 0; i < VPT; ++i) {
                    const int v = ts + ST * i;
                    if (v >= nvec) continue;
                    double* dst = p.part + (size_t)k * H + 8 * v;
#pragma unroll
                    for (int e = 0; e < 8; e += 2) {
                        double2 t;
                        t.x = (double)s_[i][e] + (double)c_[i][e];
                        t.y = (double)s_[i][e + 1] + (double)c_[i][e + 1];
                        *reinterpret_cast<double2*>(dst + e) = t;
                    }
                }
            } else {
                if (slot < nb) {
#pragma unroll
                    for (int i = 0; i < VPT; ++i) {
                        const int v = ts + ST * i;
                        if (v >= nvec) continue;
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            my64[8 * v + e] = (double)s_[i][e] + (double)c_[i][e];
                    }
                }
                __syncthreads();
                for (int col = tid; col < H; col += NT) {
                    double a = sm64[col];
                    for (int b = 1; b < nb; ++b) a += sm64[(size_t)b * nvec * 8 + col];
                    p.part[(size_t)k * H + col] = a;
                }
                __syncthreads();
            }
        }
        // let the fold kernel start its launch; it waits for this grid to finish
        asm volatile("griddepcontrol.launch_dependents;");
    } else {
        // contiguous row range of this CTA, split evenly between its slots
        const int64_t lo = (int64_t)p.R * blockIdx.x / gridDim.x;
        const int64_t hi = (int64_t)p.R * (blockIdx.x + 1) / gridDim.x;
        const int slo = (int)(lo + (hi - lo) * slot / L);
        const int shi = (int)(lo + (hi - lo) * (slot + 1) / L);
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = ts + ST * i;
            if (v < nvec)
#pragma unroll
                for (int e = 0; e < 8; ++e) my64[8 * v + e] = 0.0;
        }
        zero_state();
        constexpr int kBlock = 8;  // rows per FP32 block
        static_assert(kBlock % P == 0, "P must divide the block");
        int in_block = 0;
        for (int r = slo; r < shi; r += P) {
            do_rows(r, shi);
            in_block += P;
            if (in_block == kBlock || r + P >= shi) {
#pragma unroll
                for (int i = 0; i < VPT; ++i) {
                    const int v = ts + ST * i;
                    if (v >= nvec) continue;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        my64[8 * v + e] += (double)s_[i][e];
                        s_[i][e] = 0.f;
                    }
                }
                in_block = 0;
            }
        }
        __syncthreads();
        for (int col = tid; col < H; col += NT) {
            double a = sm64[col];
#pragma unroll
            for (int b = 1; b < L; ++b) a += sm64[(size_t)b * nvec * 8 + col];
            atomicAdd(p.acc + col, a);
        }
        __threadfence();
        __syncthreads();
        __shared__ unsigned last;
        if (tid == 0) last = (atomicAdd(p.ticket, 1u) == gridDim.x - 1) ? 1u : 0u;
        __syncthreads();
        if (last) {
            __threadfence();
            for (int col = tid; col < H; col += NT) {
                const double a = __ldcg(p.acc + col);
                p.dw[col] = __double2float_rn(a);
                p.acc[col] = 0.0;
            }
            if (tid == 0) *p.ticket = 0u;
        }
    }
}

// ============================================================================================
// Fold kernel: chunk partials -> dw, in the fixed segment order.
// ============================================================================================

constexpr int kFoldSegMax = 16;

__global__ void __launch_bounds__(32 * kFoldSegMax) bwd_fold_kernel(const BwdParams p) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    __shared__ double seg[kFoldSegMax][32];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int col = blockIdx.x * 32 + lane;
    const int nseg = p.fold_segments;
    const int n = p.n_chunks;
    const int seg_len = (n + nseg - 1) / nseg;
    if (warp < nseg && col < p.H) {
        const int k0 = warp * seg_len;
        const int k1 = min(n, k0 + seg_len);
        double a = 0.0;
        if (k0 < k1) {
            const double* src = p.part + col;
            const size_t H = (size_t)p.H;
            a = __ldcg(src + (size_t)k0 * H);
            int k = k0 + 1;
            for (; k + 8 <= k1; k += 8) {
                double t[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) t[u] = __ldcg(src + (size_t)(k + u) * H);
#pragma unroll
                for (int u = 0; u < 8; ++u) a += t[u];
            }
            for (; k < k1; ++k) a += __ldcg(src + (size_t)k * H);
        }
        seg[warp][lane] = a;
    }
    __syncthreads();
    if (warp == 0 && col < p.H) {
        double tot = seg[0][lane];
        for (int q = 1; q < nseg; ++q)
            if (q * seg_len < n) tot += seg[q][lane];
        p.dw[col] = __double2float_rn(tot);
    }
}

// ============================================================================================
// Small-row single kernel: row tasks (dx) and column tasks (dw, the full fixed order).
// ============================================================================================

constexpr int kSmallThreads = 256;
constexpr int kColStrip = 64;   // columns per column task
constexpr int kRowBatch = 16;   // rows loaded together by a column-task lane

template <int VPT, bool RES, bool W32>
__global__ void __launch_bounds__(kSmallThreads) bwd_small_kernel(const BwdParams p,
                                                                  int n_row_ctas) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int H = p.H;
    if ((int)blockIdx.x < n_row_ctas) {
        // ---- row task: one warp per row ----
        const int r = blockIdx.x * (kSmallThreads / 32) + warp;
        if (r >= p.R) return;
        const int64_t ox = row_offset(r, p.heads, p.x.st, p.x.sk);
        const int64_t ody = row_offset(r, p.heads, p.dy.st, p.dy.sk);
        const int64_t odx = row_offset(r, p.heads, p.dx.st, p.dx.sk);
        const float rs = __ldg(p.rstd + r);
        uint4 xv[VPT], dyv[VPT];
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = lane + 32 * i;
            const bool ok = v < p.nvec;
            xv[i] = ok ? ld_stream16(p.x.ptr + ox + 8 * v) : make_uint4(0u, 0u, 0u, 0u);
            dyv[i] = ok ? ld_stream16(p.dy.ptr + ody + 8 * v) : make_uint4(0u, 0u, 0u, 0u);
        }
        float d = 0.f;
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = lane + 32 * i;
            if (v >= p.nvec) continue;
            float xf[8], df[8], wf[8];
            unpack8(xv[i], xf);
            unpack8(dyv[i], df);
            load_w8<W32>(p.w, 8 * v, wf);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                d = __fmaf_rn(__fmul_rn(df[e], wf[e]), __fmul_rn(xf[e], rs), d);
        }
        const float cr = __fdiv_rn(warp_sum(d), (float)H);
        int64_t odh = 0;
        if constexpr (RES) odh = row_offset(r, p.heads, p.dh.st, p.dh.sk);
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = lane + 32 * i;
            if (v >= p.nvec) continue;
            float xf[8], df[8], wf[8], out[8];
            unpack8(xv[i], xf);
            unpack8(dyv[i], df);
            load_w8<W32>(p.w, 8 * v, wf);
            float hf[8];
            if constexpr (RES) unpack8(ld_stream16(p.dh.ptr + odh + 8 * v), hf);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float xh = __fmul_rn(xf[e], rs);
                const float g = __fmul_rn(df[e], wf[e]);
                float o = __fmul_rn(rs, __fmaf_rn(-xh, cr, g));
                if constexpr (RES) o = __fadd_rn(o, hf[e]);
                out[e] = o;
            }
            st16(p.dx.ptr + odx + 8 * v, pack8(out));
        }
        return;
    }
    // ---- column task: columns [c0, c0 + 64), every row, the whole fixed order ----
    extern __shared__ __align__(16) unsigned char smem_raw[];
    double* bp = reinterpret_cast<double*>(smem_raw);  // [n_blocks][64] block partials
    const int c0 = ((int)blockIdx.x - n_row_ctas) * kColStrip;
    const int j = c0 + 2 * lane;  // this lane's column pair
    const bool jok = j < H;
    const int B = p.block_rows;
    const int n_blocks = (p.R + B - 1) / B;
    for (int b = warp; b < n_blocks; b += kSmallThreads / 32) {
        float s0 = 0.f, k0 = 0.f, s1 = 0.f, k1 = 0.f;
        const int rb0 = b * B;
        const int rb1 = min(rb0 + B, p.R);
        for (int r = rb0; r < rb1; r += kRowBatch) {
            uint32_t xw[kRowBatch], dw2[kRowBatch];
            const float rsl = (r + lane < rb1 && lane < kRowBatch) ? __ldg(p.rstd + r + lane) : 0.f;
#pragma unroll
            for (int u = 0; u < kRowBatch; ++u) {
                const int rr = r + u;
                const bool ok = jok && rr < rb1;
                xw[u] = ok ? __ldg(reinterpret_cast<const uint32_t*>(
                                 p.x.ptr + row_offset(rr, p.heads, p.x.st, p.x.sk) + j))
                           : 0u;
                dw2[u] = ok ? __ldg(reinterpret_cast<const uint32_t*>(
                                  p.dy.ptr + row_offset(rr, p.heads, p.dy.st, p.dy.sk) + j))
                            : 0u;
            }
#pragma unroll
            for (int u = 0; u < kRowBatch; ++u) {
                const float rs = __shfl_sync(0xFFFFFFFFu, rsl, u);
                if (r + u < rb1) {
                    twosum_product(bf16lo(dw2[u]), __fmul_rn(bf16lo(xw[u]), rs), s0, k0);
                    twosum_product(bf16hi(dw2[u]), __fmul_rn(bf16hi(xw[u]), rs), s1, k1);
                }
            }
        }
        bp[(size_t)b * kColStrip + 2 * lane] = (double)s0 + (double)k0;
        bp[(size_t)b * kColStrip + 2 * lane + 1] = (double)s1 + (double)k1;
    }
    __syncthreads();
    const int t = threadIdx.x;
    if (t < kColStrip && c0 + t < H) {
        const int L = p.blocks_per_chunk;
        const int n_chunks = (n_blocks + L - 1) / L;
        const int nseg = p.fold_segments;
        const int seg_len = (n_chunks + nseg - 1) / nseg;
        double tot = 0.0;
        for (int q = 0; q < nseg; ++q) {
            const int k0c = q * seg_len;
            const int k1c = min(n_chunks, k0c + seg_len);
            if (k0c >= k1c) continue;
            double sg = 0.0;
            for (int k = k0c; k < k1c; ++k) {
                const int b0 = k * L;
                const int b1 = min(n_blocks, b0 + L);
                double ch = bp[(size_t)b0 * kColStrip + t];
                for (int b = b0 + 1; b < b1; ++b) ch += bp[(size_t)b * kColStrip + t];
                sg = (k == k0c) ? ch : sg + ch;
            }
            tot = (q == 0) ? sg : tot + sg;
        }
        p.dw[c0 + t] = __double2float_rn(tot);
    }
}

// ============================================================================================
// host side
// ============================================================================================

namespace {

template <typename K>
int occupancy(K kern, int threads, size_t smem) {
    int o = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, kern, threads, smem) != cudaSuccess)
        return 1;
    return o > 0 ? o : 1;
}

template <int SW, int VPT, int L, int P, bool DET, bool RES, bool W32>
cudaError_t launch_large(const BwdParams& p, int grid_ctas, cudaStream_t s) {
    auto kern = bwd_large_kernel<SW, VPT, L, P, DET, RES, W32>;
    constexpr int NT = SW * 32 * L;
    const size_t smem = (DET && L == 1) ? 0 : (size_t)L * p.nvec * 8 * sizeof(double);
    static int occ_cached = -1;
    static size_t smem_set = 0;
    if (smem != 0 && smem > smem_set) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        smem_set = smem;
        occ_cached = -1;
    }
    if (occ_cached < 0) occ_cached = occupancy(kern, NT, smem);
    int grid = grid_ctas;
    if (grid <= 0) {
        const int64_t cap = (int64_t)device_sm_count() * occ_cached;
        int64_t need = DET ? p.n_chunks : ((int64_t)p.R + L * 8 - 1) / (L * 8);
        if (need < 1) need = 1;
        grid = (int)(need < cap ? need : cap);
    }
    kern<<<grid, NT, smem, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || !DET) return e;
    // fold kernel, programmatic dependent launch
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((p.H + 31) / 32));
    cfg.blockDim = dim3(32 * kFoldSegMax);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, bwd_fold_kernel, p);
}

// Slot layout per width: SW warps per slot, VPT vectors per thread, L slots per CTA.
template <bool DET, bool RES, bool W32>
cudaError_t dispatch_large(const BwdParams& p, int grid_ctas, cudaStream_t s) {
    const int nv = p.nvec;
    if (nv <= 32) return launch_large<1, 1, 8, 2, DET, RES, W32>(p, grid_ctas, s);
    if (nv <= 64) return launch_large<1, 2, 8, 2, DET, RES, W32>(p, grid_ctas, s);
    if (nv <= 128) return launch_large<2, 2, 4, 2, DET, RES, W32>(p, grid_ctas, s);
    if (nv <= 192) return launch_large<2, 3, 4, 2, DET, RES, W32>(p, grid_ctas, s);
    if (nv <= 256) return launch_large<4, 2, 2, 2, DET, RES, W32>(p, grid_ctas, s);
    if (nv <= 384) return launch_large<4, 3, 2, 2, DET, RES, W32>(p, grid_ctas, s);
    if (nv <= 512) return launch_large<8, 2, 1, 2, DET, RES, W32>(p, grid_ctas, s);
    if (nv <= 768) return launch_large<8, 3, 1, 2, DET, RES, W32>(p, grid_ctas, s);
    return launch_large<8, 4, 1, 2, DET, RES, W32>(p, grid_ctas, s);
}

template <int VPT, bool RES, bool W32>
cudaError_t launch_small_t(const BwdParams& p, cudaStream_t s) {
    auto kern = bwd_small_kernel<VPT, RES, W32>;
    const int n_row_ctas = (p.R + kSmallThreads / 32 - 1) / (kSmallThreads / 32);
    const int n_col_ctas = (p.H + kColStrip - 1) / kColStrip;
    const int n_blocks = (p.R + p.block_rows - 1) / p.block_rows;
    const size_t smem = (size_t)n_blocks * kColStrip * sizeof(double);
    static size_t smem_set = 0;
    if (smem > 48 * 1024 && smem > smem_set) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        smem_set = smem;
    }
    kern<<<n_row_ctas + n_col_ctas, kSmallThreads, smem, s>>>(p, n_row_ctas);
    return cudaGetLastError();
}

template <bool RES, bool W32>
cudaError_t dispatch_small(const BwdParams& p, cudaStream_t s) {
    const int need = (p.nvec + 31) / 32;
    if (need <= 1) return launch_small_t<1, RES, W32>(p, s);
    if (need <= 2) return launch_small_t<2, RES, W32>(p, s);
    if (need <= 4) return launch_small_t<4, RES, W32>(p, s);
    if (need <= 6) return launch_small_t<6, RES, W32>(p, s);
    if (need <= 8) return launch_small_t<8, RES, W32>(p, s);
    if (need <= 12) return launch_small_t<12, RES, W32>(p, s);
    if (need <= 16) return launch_small_t<16, RES, W32>(p, s);
    if (need <= 20) return launch_small_t<20, RES, W32>(p, s);
    if (need <= 24) return launch_small_t<24, RES, W32>(p, s);
    return launch_small_t<32, RES, W32>(p, s);
}

}  // namespace

int bwd_slots_for_width(int H) {
    const int nv = H / 8;
    if (nv <= 64) return 8;
    if (nv <= 192) return 4;
    if (nv <= 384) return 2;
    return 1;
}

cudaError_t launch_bwd_small(const BwdParams& p, bool res, bool w32, cudaStream_t s) {
    if (res) return w32 ? dispatch_small<true, true>(p, s) : dispatch_small<true, false>(p, s);
    return w32 ? dispatch_small<false, true>(p, s) : dispatch_small<false, false>(p, s);
}

cudaError_t launch_bwd_det(const BwdParams& p, bool res, bool w32, int grid_ctas,
                           cudaStream_t s) {
    if (res) return w32 ? dispatch_large<true, true, true>(p, grid_ctas, s)
                        : dispatch_large<true, true, false>(p, grid_ctas, s);
    return w32 ? dispatch_large<true, false, true>(p, grid_ctas, s)
               : dispatch_large<true, false, false>(p, grid_ctas, s);
}

cudaError_t launch_bwd_nondet(const BwdParams& p, bool res, bool w32, int grid_ctas,
                              cudaStream_t s) {
    if (res) return w32 ? dispatch_large<false, true, true>(p, grid_ctas, s)
                        : dispatch_large<false, true, false>(p, grid_ctas, s);
    return w32 ? dispatch_large<false, false, true>(p, grid_ctas, s)
               : dispatch_large<false, false, false>(p, grid_ctas, s);
}

}  // namespace rmsk
