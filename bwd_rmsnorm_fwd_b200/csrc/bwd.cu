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
//   grid or on the SM count.  Two programs produce exactly these bits:
//     - bwd_small_kernel: one launch; row tasks compute dx, column tasks walk every
//       row of a 64-column strip and do the whole fold (used for small row counts);
//     - bwd_staged_kernel<DET> + bwd_fold_kernel: CTAs take whole chunks (each slot of
//       the CTA one block), write FP64 chunk partials to the workspace, and the fold
//       kernel (launched with programmatic dependent launch) finishes the order.
// * non-deterministic: every thread sums eight rows at a time in FP32 (one FMA per
//   element) and adds each eight-row block into FP64 registers; a CTA's totals meet in
//   shared memory and the CTA adds them into an FP64 workspace vector with atomics.  The last CTA to finish (atomic ticket) rounds the
//   vector to FP32 dw and clears it for the next call.
//
// The large kernel gives each CTA L "slots" of ST consumer threads; a slot owns one row at
// a time and every thread of the slot owns VPT 16-byte column vectors, so the dw state of
// a column stays in one thread's registers for the whole block.  The per-row dot
// product is a warp-shuffle tree plus, for multi-warp slots, a named barrier over the
// slot's warps with a double-buffered shared exchange.
#include "common.cuh"

namespace rmsk {

__device__ __forceinline__ void named_bar(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Sums of P values over each group of G consecutive lanes at once (G a power of two <= 32,
// P in {1, 2, 4}, P <= G): a butterfly whose first levels exchange halves of the value set
// instead of whole values, so P sums cost about as many shuffles as one.  Lane l of a group
// returns the sum of value q = (l % G) / (G / P).
template <int G, int P>
__device__ __forceinline__ float multi_sum(const float (&v)[P], int lane) {
    static_assert(P == 1 || P == 2 || P == 4, "one, two or four values");
    static_assert(P <= G && (G & (G - 1)) == 0 && G <= 32, "whole lane groups");
    constexpr unsigned kAll = 0xFFFFFFFFu;
    if constexpr (P == 1) {
        return group_sum<G>(v[0]);
    } else if constexpr (P == 2) {
        const bool hi = (lane & (G / 2)) != 0;
        float a = (hi ? v[1] : v[0]) + __shfl_xor_sync(kAll, hi ? v[0] : v[1], G / 2);
#pragma unroll
        for (int o = G / 4; o > 0; o >>= 1) a += __shfl_xor_sync(kAll, a, o);
        return a;
    } else {
        const bool hi = (lane & (G / 2)) != 0;
        // a0 holds value (hi ? 2 : 0), a1 value (hi ? 3 : 1), each over a lane pair
        const float a0 = (hi ? v[2] : v[0]) + __shfl_xor_sync(kAll, hi ? v[0] : v[2], G / 2);
        const float a1 = (hi ? v[3] : v[1]) + __shfl_xor_sync(kAll, hi ? v[1] : v[3], G / 2);
        const bool mid = (lane & (G / 4)) != 0;
        float b = (mid ? a1 : a0) + __shfl_xor_sync(kAll, mid ? a0 : a1, G / 4);
#pragma unroll
        for (int o = G / 8; o > 0; o >>= 1) b += __shfl_xor_sync(kAll, b, o);
        return b;
    }
}

// The P row dot products of a slot of ST threads, one row at a time: a shuffle tree per row,
// then (slots of several warps) one partial per (row, warp) behind the slot's named barrier
// and a second tree over them.  Measured faster than slot_dots for the blocked-FP32 consumer
// when one multi-warp slot fills the CTA.
template <int ST, int P>
__device__ __forceinline__ void slot_dots_rowwise(const float (&v)[P], float (&dot)[P], float* red,
                                                  int slot, int buf, int lane, int wis) {
    constexpr int G = ST < 32 ? ST : 32;
    constexpr int SW = ST >= 32 ? ST / 32 : 1;
#pragma unroll
    for (int q = 0; q < P; ++q) dot[q] = group_sum<G>(v[q]);
    if constexpr (SW > 1) {
        float* r = red + (size_t)(slot * 2 + buf) * P * SW;
        if (lane == 0) {
#pragma unroll
            for (int q = 0; q < P; ++q) r[q * SW + wis] = dot[q];
        }
        named_bar(1 + slot, ST);
#pragma unroll
        for (int q = 0; q < P; ++q) dot[q] = warp_sum(lane < SW ? r[q * SW + lane] : 0.f);
    }
}

// The P row dot products of a slot of ST threads (a few lanes of a warp, one warp, or SW
// warps): every thread passes its partial sums and receives the slot's totals.  Across
// warps, one partial per (row, warp) meets in the shared buffer `red` ([L][2][P][SW],
// double-buffered by `buf`) behind the slot's named barrier, and one lane group per row
// adds them.
template <int ST, int P>
__device__ __forceinline__ void slot_dots(const float (&v)[P], float (&dot)[P], float* red,
                                          int slot, int buf, int lane, int wis) {
    constexpr unsigned kAll = 0xFFFFFFFFu;
    constexpr int G = ST < 32 ? ST : 32;
    constexpr int SW = ST >= 32 ? ST / 32 : 1;
    constexpr int GP = G / P;  // lanes per row after the butterfly
    const float mine = multi_sum<G, P>(v, lane);
    if constexpr (SW == 1) {
        const int base = lane & ~(G - 1);
#pragma unroll
        for (int q = 0; q < P; ++q) dot[q] = __shfl_sync(kAll, mine, base + q * GP);
    } else {
        float* r = red + (size_t)(slot * 2 + buf) * P * SW;
        if (lane % GP == 0) r[(lane / GP) * SW + wis] = mine;
        named_bar(1 + slot, ST);
        const int q = lane / GP;
        float a = 0.f;
#pragma unroll
        for (int w = lane % GP; w < SW; w += GP) a += r[q * SW + w];
#pragma unroll
        for (int o = GP / 2; o > 0; o >>= 1) a += __shfl_xor_sync(kAll, a, o);
#pragma unroll
        for (int qq = 0; qq < P; ++qq) dot[qq] = __shfl_sync(kAll, a, qq * GP);
    }
}

// ============================================================================================
// Large-row kernel: a bulk-copy pipeline.  Warp 0 streams the rows of each tile (x, dy
// and, in the residual form, dh) into a ring of shared-memory stages with cp.async.bulk,
// one mbarrier per stage counting the bytes; the consumer warps read the stage, compute
// dx and accumulate dw, and release the stage on a second mbarrier.  The bytes in flight
// are bounded by shared memory (up to ~200 KB per SM), not by registers.
//
// Tiles: a tile holds P consecutive rows of every slot.  Deterministic: CTA c takes chunks
// c, c + grid, ...; slot s of chunk k owns the block of rows [k*L*B + s*B, +B).
// Non-deterministic: CTA c takes a contiguous row range, split evenly between slots.
//
// Every wait is bounded (BwdParams::wait_cycles).  A wait that gives up sets the status
// word and a CTA-wide abort flag; from then on consumers stop waiting (control flow stays
// uniform, so every named barrier is still met) and the producer issues nothing more,
// then waits for its copies in flight before the CTA exits.
// ============================================================================================

// Blocked-FP32 finish, run by the last CTA to take a ticket: the FP64 column totals become dw
// and are cleared for the next call.  The loads go out in batches: the stores to dw and to
// the totals may alias later loads as far as the compiler knows, so a plain per-column loop
// would wait one L2 round trip per column (24 in a row at H 6144 with 256 threads).
constexpr int kFinishBatch = 8;

__device__ __forceinline__ void finish_dw(const BwdParams& p, int tid, int nt) {
    const int H = p.H;
    for (int c0 = tid; c0 < H; c0 += kFinishBatch * nt) {
        double tot[kFinishBatch];
        float prev[kFinishBatch];
#pragma unroll
        for (int u = 0; u < kFinishBatch; ++u) {
            const int c = c0 + u * nt;
            tot[u] = c < H ? __ldcg(p.acc + c) : 0.0;
            prev[u] = (p.accumulate && c < H) ? __ldcg(p.dw + c) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kFinishBatch; ++u) {
            const int c = c0 + u * nt;
            if (c < H) {
                const float v = __double2float_rn(tot[u]);
                p.dw[c] = p.accumulate ? __fadd_rn(prev[u], v) : v;
                p.acc[c] = 0.0;
            }
        }
    }
}

constexpr int kMaxStages = 16;
constexpr int kStagedHeader = 2048;  // barriers, flags, slot reduction buffers

struct StagedCfg {
    int32_t n_stages;
    int32_t stage_bytes;   // one stage, all tensors
    int32_t tensor_bytes;  // one tensor's rows inside a stage
    int32_t xch_offset;    // FP64 exchange of a chunk's blocks: [xch_rows][nvec*8]
    int32_t xch_rows;      // L: every block its own row, one barrier (short blocks);
                           // 1: a running sum in block order (64-row blocks, frees a stage)
    int32_t stage_offset;
};

// Rows of the deterministic chunk exchange: one row per block for blocks shorter than 64 rows
// (a chunk there is only a few tiles, and one barrier per block would dominate: [1024,24,256]
// 31.2 vs 25.1 us), a single running-sum row for 64-row blocks (the smaller exchange leaves
// room for one more pipeline stage: H 512 x 131072 93 vs 101 us, H 1536 x 65537 124 vs 134 us).
inline int det_xch_rows(bool det, int L, int block_rows) {
    if (!det || L == 1) return 0;
    return block_rows < 64 ? L : 1;
}

template <int ST, int VPT, int L, int P, bool DET, int NV, bool RES, bool W32, int MINB>
__global__ void __launch_bounds__(32 + ST * L, MINB)
    bwd_staged_kernel(const BwdParams p, const StagedCfg sc, const __grid_constant__ RowMaps tm) {
    // NV != 0: the width is exactly NV vectors, every consumer thread owns VPT of them, and
    // the row size is a compile-time constant (no per-vector range checks, constant offsets)
    static_assert(NV == 0 || NV == ST * VPT, "a whole-width layout owns every vector");
    // ST threads per slot: a few lanes of a warp (8 or 16: several rows per warp), one warp,
    // or several warps (a named barrier joins them)
    static_assert(ST >= 32 ? ST % 32 == 0 : 32 % ST == 0, "slot must tile warps");
    static_assert((ST * L) % 32 == 0, "consumers must fill whole warps");
    constexpr int SW = ST >= 32 ? ST / 32 : 1;  // warps per slot
    constexpr int NCW = ST * L / 32;            // consumer warps
    constexpr int NCT = NCW * 32;    // consumer threads
    constexpr int RT = L * P;        // rows per stage
    constexpr int NTEN = RES ? 3 : 2;
    constexpr int kAllConsumers = 15;  // named barrier over every consumer thread
    static_assert(16 * kMaxStages + 16 + (ST > 32 ? L * 2 * P * SW * 4 : 0) <= kStagedHeader,
                  "slot reduction buffers must fit in the header");
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);  // full[kMaxStages], empty[kMaxStages]
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + 16 * kMaxStages);
    volatile unsigned* last_flag = reinterpret_cast<volatile unsigned*>(smem + 16 * kMaxStages + 4);
    float* red = reinterpret_cast<float*>(smem + 16 * kMaxStages + 16);  // [L][2][P][SW]
    double* xch = reinterpret_cast<double*>(smem + sc.xch_offset);       // [xch_rows][nvec*8]
    unsigned char* stages = smem + sc.stage_offset;

    const int NS = sc.n_stages;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int H = NV ? NV * 8 : p.H;
    const int nvec = NV ? NV : p.nvec;
    const uint32_t row_bytes = (uint32_t)nvec * 16u;
    const int64_t limit = p.wait_cycles;
    auto full_bar = [&](int s) { return smem_addr(&bars[s]); };
    auto empty_bar = [&](int s) { return smem_addr(&bars[kMaxStages + s]); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), NCW);
        }
        *abort_flag = 0;
        *last_flag = 0;
        mbar_init_fence();
    }
    __syncthreads();

    // ---- the unit sequence (chunks or the CTA's row range), identical for all warps ----
    const int B = p.block_rows;
    const int CH = B * L;
    int64_t lo = 0, hi = 0;
    if constexpr (!DET) {
        lo = (int64_t)p.R * blockIdx.x / gridDim.x;
        hi = (int64_t)p.R * (blockIdx.x + 1) / gridDim.x;
    }
    const int n_units = DET ? (p.n_chunks > (int)blockIdx.x
                                   ? (p.n_chunks - 1 - (int)blockIdx.x) / (int)gridDim.x + 1
                                   : 0)
                            : 1;
    // first row and end row of slot s in unit u
    auto slot_base = [&](int u, int s) -> int {
        if constexpr (DET) {
            const int k = (int)blockIdx.x + u * (int)gridDim.x;
            return k * CH + s * B;
        } else {
            return (int)(lo + (hi - lo) * s / L);
        }
    };
    auto slot_end = [&](int u, int s) -> int {
        if constexpr (DET) {
            return min(slot_base(u, s) + B, p.R);
        } else {
            return (int)(lo + (hi - lo) * (s + 1) / L);
        }
    };
    auto unit_tiles = [&](int u) -> int {
        int m = 0;
#pragma unroll
        for (int s = 0; s < L; ++s) m = max(m, slot_end(u, s) - slot_base(u, s));
        return (m + P - 1) / P;
    };

    if (warp == 0) {
        // ================= producer =================
        // tensor loads also need a 128-byte aligned destination (checked once, used for both
        // the byte count and the copies)
        const bool tma_ok = (smem_addr(stages) & 127u) == 0 && (row_bytes & 127u) == 0;
        int j = 0;
        for (int u = 0; u < n_units; ++u) {
            const int nt = unit_tiles(u);
            for (int t = 0; t < nt; ++t, ++j) {
                const int stage = j % NS;
                const uint32_t ph = (uint32_t)(j / NS) & 1u;
                if (j >= NS) {
                    if (!mbar_wait_bounded(empty_bar(stage), ph ^ 1u, limit)) {
                        if (lane == 0) { *abort_flag = 1; atomicOr(p.status, kStatusTimeout); }
                    }
                }
                __syncwarp();
                if (*abort_flag) goto drain;
                uint32_t bytes = 0;  // a TMA box always lands whole (rows past the end as 0)
#pragma unroll
                for (int s = 0; s < L; ++s) {
                    const int n = min(P, slot_end(u, s) - (slot_base(u, s) + t * P));
                    if (n > 0)
#pragma unroll
                        for (int ten = 0; ten < NTEN; ++ten)
                            bytes += (uint32_t)(tm.use[ten] && tma_ok ? P : n) * row_bytes;
                }
                if (lane == 0) mbar_arrive_expect_tx(full_bar(stage), bytes);
                __syncwarp();
                const uint32_t sbase = smem_addr(stages + (size_t)stage * sc.stage_bytes);
                // one TMA box per (tensor, slot) for equally spaced rows of H <= 256, one bulk
                // copy per (tensor, slot) for contiguous rows, else one bulk copy per row
                for (int c = lane; c < L * NTEN; c += 32) {
                    const int ten = c / L;
                    const int s = c - ten * L;
                    const RowsIn& src = ten == 0 ? p.x : (ten == 1 ? p.dy : p.dh);
                    const int row0 = slot_base(u, s) + t * P;
                    const int n = min(P, slot_end(u, s) - row0);
                    if (n <= 0) continue;
                    const uint32_t dst =
                        sbase + (uint32_t)ten * sc.tensor_bytes + (uint32_t)(s * P) * row_bytes;
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
                    const int row = slot_base(u, s) + t * P + q;
                    const RowsIn& src = ten == 0 ? p.x : (ten == 1 ? p.dy : p.dh);
                    if (row < slot_end(u, s) && !(tm.use[ten] && tma_ok) && !rows_contiguous(src, p.heads, H)) {
                        bulk_load(sbase + (uint32_t)ten * sc.tensor_bytes + (uint32_t)rr * row_bytes,
                                  src.ptr + row_offset(row, p.heads, src.st, src.sk), row_bytes,
                                  full_bar(stage));
                    }
                }
                __syncwarp();
            }
        }
    drain:
        // every copy issued lands before the CTA may exit (bounded, with the default
        // limit even when a shorter one was requested)
        if (lane == 0) {
            const int last = j;  // tiles issued
            for (int i = 0; i < NS && i < last; ++i) {
                const int jj = last - 1 - i;
                mbar_wait_bounded(full_bar(jj % NS), (uint32_t)(jj / NS) & 1u,
                                  limit > kDefaultWaitCycles ? limit : kDefaultWaitCycles);
            }
        }
        return;
    }

    // ================= consumers =================
    // Packed-pair arithmetic on -xh: every product is formed with nx = x * (-rstd), which
    // is exactly -xh (round-to-nearest is sign-symmetric), so the deterministic TwoSum
    // state holds exactly the negation of the documented order's state and is negated
    // back when a block is converted to FP64.
    const int ctid = threadIdx.x - 32;
    const int slot = ctid / ST;
    const int ts = ctid - slot * ST;
    const int wis = ts >> 5;
    const float invH = 1.0f / (float)H;
    const float2 m1 = make_float2(-1.f, -1.f);

    float2 w2[VPT][4];
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int v = ts + ST * i;
        float wf[8];
        if (NV || v < nvec) {
            load_w8<W32>(p.w, 8 * v, wf);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) wf[e] = 0.f;
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) w2[i][k] = make_float2(wf[2 * k], wf[2 * k + 1]);
    }
    // DET: (s, c) TwoSum state of -dw.  NONDET: s = eight-row FP32 block of -dw and acc,
    // the FP64 total of dw.
    float2 s2[VPT][4], c2[VPT][DET ? 4 : 1];
    double acc[DET ? 1 : VPT][DET ? 1 : 8];
    if constexpr (!DET) {
#pragma unroll
        for (int i = 0; i < VPT; ++i)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[i][e] = 0.0;
    }
    int buf = 0;
    int j = 0;
    int in_block = 0;
    // rstd of the next tile, loaded one tile ahead
    float rs_next[P];
    {
        const int b0 = n_units > 0 ? slot_base(0, slot) : 0;
        const int e0 = n_units > 0 ? slot_end(0, slot) : 0;
#pragma unroll
        for (int q = 0; q < P; ++q) rs_next[q] = (b0 + q < e0) ? __ldg(p.rstd + b0 + q) : 0.f;
    }
    for (int u = 0; u < n_units; ++u) {
        const int base = slot_base(u, slot);
        const int endr = slot_end(u, slot);
        const int nt = unit_tiles(u);
#pragma unroll
        for (int i = 0; i < VPT; ++i)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                s2[i][k] = make_float2(0.f, 0.f);
                if constexpr (DET) c2[i][k] = make_float2(0.f, 0.f);
            }
        for (int t = 0; t < nt; ++t, ++j) {
            const int stage = j % NS;
            const uint32_t ph = (uint32_t)(j / NS) & 1u;
            float rs[P];
#pragma unroll
            for (int q = 0; q < P; ++q) rs[q] = rs_next[q];
            {   // prefetch the next tile's rstd (next unit's first tile at the end of a unit)
                int nb = base + (t + 1) * P, ne = endr;
                if (t + 1 == nt) {
                    nb = u + 1 < n_units ? slot_base(u + 1, slot) : 0;
                    ne = u + 1 < n_units ? slot_end(u + 1, slot) : 0;
                }
#pragma unroll
                for (int q = 0; q < P; ++q) rs_next[q] = (nb + q < ne) ? __ldg(p.rstd + nb + q) : 0.f;
            }
            if (!*abort_flag) {
                if (!mbar_wait_bounded(full_bar(stage), ph, limit)) {
                    *abort_flag = 1;
                    if (lane == 0) atomicOr(p.status, kStatusTimeout);
                }
            }
            const unsigned char* sb = stages + (size_t)stage * sc.stage_bytes;
            const uint4* sx = reinterpret_cast<const uint4*>(sb + (size_t)(slot * P) * row_bytes);
            const uint4* sdy = reinterpret_cast<const uint4*>(sb + sc.tensor_bytes +
                                                              (size_t)(slot * P) * row_bytes);
            const uint4* sdh = reinterpret_cast<const uint4*>(sb + 2 * sc.tensor_bytes +
                                                              (size_t)(slot * P) * row_bytes);
            if constexpr (DET && ST <= 32) {
                // deterministic slots within one warp: one row at a time.  Each 16-byte vector
                // is unpacked once and kept in registers through both passes, and the row's
                // dot is one tree over the slot's lanes (every lane takes part in every row's
                // shuffles; rows past the slot's end are skipped after them).  Measured against
                // the two passes below: H 256 x 1M 303 vs 319 us, H 512 x 65536 56.6 vs 59.7
                // us, [16384,4,256] 31.3 vs 33.6 us, [1024,24,256] 20.0 vs 21.3 us; same dw
                // bits.  The blocked-FP32 consumer measured 1-2 % slower this way and keeps the
                // two passes.
#pragma unroll
                for (int q = 0; q < P; ++q) {
                    float2 xf[VPT][4], df[VPT][4];
                    float2 d2 = make_float2(0.f, 0.f);
#pragma unroll
                    for (int i = 0; i < VPT; ++i) {
                        const int v = ts + ST * i;
                        const bool in = NV || v < nvec;
                        const uint4 xr = in ? sx[q * nvec + v] : make_uint4(0u, 0u, 0u, 0u);
                        const uint4 dr = in ? sdy[q * nvec + v] : make_uint4(0u, 0u, 0u, 0u);
                        const uint32_t xw[4] = {xr.x, xr.y, xr.z, xr.w};
                        const uint32_t dw4[4] = {dr.x, dr.y, dr.z, dr.w};
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            xf[i][k] = bf16x2_to_f2(xw[k]);
                            df[i][k] = bf16x2_to_f2(dw4[k]);
                            d2 = fma2(mul2(df[i][k], w2[i][k]), xf[i][k], d2);
                        }
                    }
                    const float dotq = group_sum<ST>((d2.x + d2.y) * -rs[q]);
                    if (base + t * P + q >= endr) continue;
                    const float cr = -dotq * invH;
                    const float2 c2v = make_float2(cr, cr);
                    const float2 rs2 = make_float2(rs[q], rs[q]);
                    const float2 nrs = make_float2(-rs[q], -rs[q]);
                    const int row = base + t * P + q;
                    uint16_t* dxrow = p.dx.ptr + row_offset(row, p.heads, p.dx.st, p.dx.sk);
#pragma unroll
                    for (int i = 0; i < VPT; ++i) {
                        const int v = ts + ST * i;
                        if (!NV && v >= nvec) continue;
                        uint32_t hw[4] = {0u, 0u, 0u, 0u};
                        if constexpr (RES) {
                            const uint4 hr = sdh[q * nvec + v];
                            hw[0] = hr.x; hw[1] = hr.y; hw[2] = hr.z; hw[3] = hr.w;
                        }
                        uint32_t out[4];
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const float2 d = df[i][k];
                            const float2 nx = mul2(xf[i][k], nrs);
                            const float2 g = mul2(d, w2[i][k]);
                            float2 o = mul2(fma2(nx, c2v, g), rs2);
                            if constexpr (RES) o = add2(o, bf16x2_to_f2(hw[k]));
                            out[k] = pack2(o);
                            const float2 np = mul2(d, nx);
                            const float2 ne = make_float2(__fmaf_rn(d.x, nx.x, -np.x),
                                                          __fmaf_rn(d.y, nx.y, -np.y));
                            const float2 tt = add2(s2[i][k], np);
                            const float2 z = sub2(tt, s2[i][k]);
                            const float2 err = add2(sub2(s2[i][k], sub2(tt, z)), sub2(np, z));
                            c2[i][k] = add2(c2[i][k], add2(err, ne));
                            s2[i][k] = tt;
                        }
                        st16(dxrow + 8 * v, make_uint4(out[0], out[1], out[2], out[3]));
                    }
                }
            } else {
                // pass 1: per-thread partial sums of g * x, scaled by -rstd once per row to give
                // the partial sums of g * (-xh) (one packed multiply per pair fewer than forming
                // -xh here; the dot only enters dx)
                float dpart[P], dot[P];
#pragma unroll
                for (int q = 0; q < P; ++q) {
                    float2 d2 = make_float2(0.f, 0.f);
#pragma unroll
                    for (int i = 0; i < VPT; ++i) {
                        const int v = ts + ST * i;
                        if (NV || v < nvec) {
                            const uint4 xr = sx[q * nvec + v];
                            const uint4 dr = sdy[q * nvec + v];
                            const uint32_t xw[4] = {xr.x, xr.y, xr.z, xr.w};
                            const uint32_t dw4[4] = {dr.x, dr.y, dr.z, dr.w};
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                d2 = fma2(mul2(bf16x2_to_f2(dw4[k]), w2[i][k]),
                                          bf16x2_to_f2(xw[k]), d2);
                        }
                    }
                    dpart[q] = (d2.x + d2.y) * -rs[q];
                }
                // the blocked-FP32 consumer of one multi-warp slot per CTA reduces row by row
                // (measured faster there: H 4096-6144); every other layout takes the multi-row
                // butterfly (H 2048 blocked FP32 with two slots: 137 vs 162 us)
                if constexpr (DET || SW == 1 || L > 1)
                    slot_dots<ST, P>(dpart, dot, red, slot, buf, lane, wis);
                else
                    slot_dots_rowwise<ST, P>(dpart, dot, red, slot, buf, lane, wis);
                if constexpr (SW > 1) buf ^= 1;
                // pass 2: dx = rstd (g - xh c) = rstd (g + nx c), c = -dot / H; dw, rows in order
#pragma unroll
                for (int q = 0; q < P; ++q) {
                    if (base + t * P + q >= endr) continue;
                    const float cr = -dot[q] * invH;
                    const float2 c2v = make_float2(cr, cr);
                    const float2 rs2 = make_float2(rs[q], rs[q]);
                    const float2 nrs = make_float2(-rs[q], -rs[q]);
                    const int row = base + t * P + q;
                    uint16_t* dxrow = p.dx.ptr + row_offset(row, p.heads, p.dx.st, p.dx.sk);
#pragma unroll
                    for (int i = 0; i < VPT; ++i) {
                        const int v = ts + ST * i;
                        if (!NV && v >= nvec) continue;
                        const uint4 xr = sx[q * nvec + v];
                        const uint4 dr = sdy[q * nvec + v];
                        const uint32_t xw[4] = {xr.x, xr.y, xr.z, xr.w};
                        const uint32_t dw4[4] = {dr.x, dr.y, dr.z, dr.w};
                        uint32_t hw[4] = {0u, 0u, 0u, 0u};
                        if constexpr (RES) {
                            const uint4 hr = sdh[q * nvec + v];
                            hw[0] = hr.x; hw[1] = hr.y; hw[2] = hr.z; hw[3] = hr.w;
                        }
                        uint32_t out[4];
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const float2 d = bf16x2_to_f2(dw4[k]);
                            const float2 nx = mul2(bf16x2_to_f2(xw[k]), nrs);
                            const float2 g = mul2(d, w2[i][k]);
                            float2 o = mul2(fma2(nx, c2v, g), rs2);
                            if constexpr (RES) o = add2(o, bf16x2_to_f2(hw[k]));
                            out[k] = pack2(o);
                            if constexpr (DET) {
                                // -p and its exact error -e = fma(d, -xh, p) (two scalar FMAs with
                                // a negated addend: cheaper than a packed negation), then TwoSum;
                                // err + (-e) rounds exactly as err - e
                                const float2 np = mul2(d, nx);
                                const float2 ne = make_float2(__fmaf_rn(d.x, nx.x, -np.x),
                                                              __fmaf_rn(d.y, nx.y, -np.y));
                                const float2 tt = add2(s2[i][k], np);
                                const float2 z = sub2(tt, s2[i][k]);
                                const float2 err = add2(sub2(s2[i][k], sub2(tt, z)), sub2(np, z));
                                c2[i][k] = add2(c2[i][k], add2(err, ne));
                                s2[i][k] = tt;
                            } else {
                                s2[i][k] = fma2(d, nx, s2[i][k]);
                            }
                        }
                        st16(dxrow + 8 * v, make_uint4(out[0], out[1], out[2], out[3]));
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty_bar(stage));
            if constexpr (!DET) {
                // eight-row FP32 blocks go into the FP64 total
                in_block += P;
                if (in_block >= 8 || t + 1 == nt) {
#pragma unroll
                    for (int i = 0; i < VPT; ++i)
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            acc[i][2 * k] -= (double)s2[i][k].x;
                            acc[i][2 * k + 1] -= (double)s2[i][k].y;
                            s2[i][k] = make_float2(0.f, 0.f);
                        }
                    in_block = 0;
                }
            }
        }
        if constexpr (DET) {
            const int k = (int)blockIdx.x + u * (int)gridDim.x;
            const int nb = min(L, (p.R - k * CH + B - 1) / B);  // non-empty blocks of chunk k
            if constexpr (L == 1) {
#pragma unroll
                for (int i = 0; i < VPT; ++i) {
                    const int v = ts + ST * i;
                    if (!NV && v >= nvec) continue;
                    double* dst = p.part + (size_t)k * H + 8 * v;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        double2 t2;
                        t2.x = -((double)s2[i][kk].x + (double)c2[i][kk].x);
                        t2.y = -((double)s2[i][kk].y + (double)c2[i][kk].y);
                        *reinterpret_cast<double2*>(dst + 2 * kk) = t2;
                    }
                }
            } else if (sc.xch_rows > 1) {
                // every block to its own FP64 row, one consumer barrier, then each column's
                // blocks folded left to right
                if (slot < nb) {
#pragma unroll
                    for (int i = 0; i < VPT; ++i) {
                        const int v = ts + ST * i;
                        if (!NV && v >= nvec) continue;
                        double* mine = xch + (size_t)slot * nvec * 8 + 8 * v;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            mine[2 * kk] = -((double)s2[i][kk].x + (double)c2[i][kk].x);
                            mine[2 * kk + 1] = -((double)s2[i][kk].y + (double)c2[i][kk].y);
                        }
                    }
                }
                named_bar(kAllConsumers, NCT);
                for (int col = ctid; col < H; col += NCT) {
                    double a = xch[col];
                    for (int b = 1; b < nb; ++b) a += xch[(size_t)b * nvec * 8 + col];
                    p.part[(size_t)k * H + col] = a;
                }
                named_bar(kAllConsumers, NCT);
            } else {
                // the chunk's blocks folded left to right through one FP64 row: slot b adds
                // its block to the running sum after slot b - 1 has (one consumer barrier per
                // block), and the last block's slot stores the chunk partial
                for (int b = 0; b < nb; ++b) {
                    if (slot == b) {
#pragma unroll
                        for (int i = 0; i < VPT; ++i) {
                            const int v = ts + ST * i;
                            if (!NV && v >= nvec) continue;
                            double* run = xch + 8 * v;
                            double* dst = p.part + (size_t)k * H + 8 * v;
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                double2 t2;
                                t2.x = -((double)s2[i][kk].x + (double)c2[i][kk].x);
                                t2.y = -((double)s2[i][kk].y + (double)c2[i][kk].y);
                                if (b > 0) {
                                    t2.x = run[2 * kk] + t2.x;
                                    t2.y = run[2 * kk + 1] + t2.y;
                                }
                                if (b + 1 < nb) {
                                    run[2 * kk] = t2.x;
                                    run[2 * kk + 1] = t2.y;
                                } else {
                                    *reinterpret_cast<double2*>(dst + 2 * kk) = t2;
                                }
                            }
                        }
                    }
                    named_bar(kAllConsumers, NCT);
                }
            }
        }
    }
    if constexpr (DET) {
        // let the fold kernel begin launching; it waits for this grid to complete
        asm volatile("griddepcontrol.launch_dependents;");
    } else {
        // slot totals meet in shared memory (the stage ring, free once every tile is
        // consumed), then one FP64 atomic per column per CTA
        double* tot = reinterpret_cast<double*>(stages);
        named_bar(kAllConsumers, NCT);
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = ts + ST * i;
            if (!NV && v >= nvec) continue;
#pragma unroll
            for (int e = 0; e < 8; ++e) tot[(size_t)slot * nvec * 8 + 8 * v + e] = acc[i][e];
        }
        named_bar(kAllConsumers, NCT);
        for (int col = ctid; col < H; col += NCT) {
            double a = tot[col];
#pragma unroll
            for (int b = 1; b < L; ++b) a += tot[(size_t)b * nvec * 8 + col];
            atomicAdd(p.acc + col, a);
        }
        __threadfence();
        named_bar(kAllConsumers, NCT);
        if (ctid == 0) *last_flag = (atomicAdd(p.ticket, 1u) == gridDim.x - 1) ? 1u : 0u;
        named_bar(kAllConsumers, NCT);
        if (*last_flag) {
            __threadfence();
            finish_dw(p, ctid, NCT);
            if (ctid == 0) *p.ticket = 0u;
        }
    }
}

// ============================================================================================
// Narrow-row kernel for mid-sized blocked-FP32 backwards (H <= 512, R*H < 2^24): one warp per
// row, no producer warp and no barrier on the data path.  Lane l owns the column vectors l and
// l + 32 of every row, so its dw state never leaves registers.  Each warp runs its own
// S-stage ring in shared memory, filled with per-lane cp.async: lane l copies its own 16-byte
// vectors of x, dy (and dh) and the row's rstd S-1 rows ahead and later reads back only what
// it copied itself, so a per-thread cp.async.wait_group is all the synchronisation the ring
// needs.  With no pipeline to fill and drain per CTA it finishes small problems sooner than
// the bulk-copy kernel; on large ones it issues about 1.8x the instructions per row (a lane
// holds only 8 or 16 elements of a row) and the bulk-copy kernel is faster, so it is used
// below 2^24 elements only.  Rows are taken grid-stride; eight-row FP32 blocks go into FP64
// registers; the warp totals meet in shared memory, then one FP64 atomic per column per CTA
// and the last-CTA ticket, as in the bulk-copy kernel.
// ============================================================================================

constexpr int kWarpBwdWarps = 8;
constexpr int64_t kWarpBwdMaxElems = int64_t(1) << 24;

// Bytes of one ring stage of one warp: NTEN tensors x VPT vectors x 32 lanes x 16 bytes, then
// 32 lanes x 4 bytes of rstd.
template <int VPT, bool RES>
__host__ __device__ constexpr int warp_stage_bytes() {
    return (RES ? 3 : 2) * VPT * 32 * 16 + 32 * 4;
}

template <int VPT, int S, bool RES, bool W32>
__global__ void __launch_bounds__(32 * kWarpBwdWarps) bwd_warp_kernel(const BwdParams p) {
    constexpr int NTEN = RES ? 3 : 2;
    constexpr int SB = warp_stage_bytes<VPT, RES>();
    constexpr int nw = kWarpBwdWarps;
    extern __shared__ __align__(16) unsigned char wsmem[];
    __shared__ unsigned last;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int H = p.H;
    const int nvec = p.nvec;
    const float invH = 1.0f / (float)H;
    double* tot = reinterpret_cast<double*>(wsmem);  // [warps][H]
    unsigned char* ring = wsmem + (size_t)nw * H * sizeof(double) + (size_t)warp * S * SB;
    const uint32_t ring_s = smem_addr(ring);

    float2 w2[VPT][4];
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int v = lane + 32 * i;
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
    // s = eight-row FP32 block of -dw, acc = FP64 total of dw
    float2 s2[VPT][4];
    double acc[VPT][8];
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
#pragma unroll
        for (int k = 0; k < 4; ++k) s2[i][k] = make_float2(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[i][e] = 0.0;
    }

    // the warp's rows: gw, gw + (warps in the grid), ...
    const int gw = blockIdx.x * nw + warp;
    const int nwt = gridDim.x * nw;
    const int total = p.R > gw ? (p.R - 1 - gw) / nwt + 1 : 0;
    auto issue = [&](int j) {
        if (j < total) {
            const int r = gw + j * nwt;
            const uint32_t st = ring_s + (uint32_t)((j % S) * SB);
            const int64_t ox = row_offset(r, p.heads, p.x.st, p.x.sk);
            const int64_t od = row_offset(r, p.heads, p.dy.st, p.dy.sk);
            const int64_t oh = RES ? row_offset(r, p.heads, p.dh.st, p.dh.sk) : 0;
#pragma unroll
            for (int i = 0; i < VPT; ++i) {
                const int v = lane + 32 * i;
                if (v < nvec) {
                    cp_async16(st + (uint32_t)((0 * VPT + i) * 512 + lane * 16), p.x.ptr + ox + 8 * v);
                    cp_async16(st + (uint32_t)((1 * VPT + i) * 512 + lane * 16), p.dy.ptr + od + 8 * v);
                    if constexpr (RES)
                        cp_async16(st + (uint32_t)((2 * VPT + i) * 512 + lane * 16), p.dh.ptr + oh + 8 * v);
                }
            }
            cp_async4(st + (uint32_t)(NTEN * VPT * 512 + lane * 4), p.rstd + r);
        }
        cp_async_commit();  // one group per row, empty or not: wait_group counts them
    };

#pragma unroll
    for (int j = 0; j < S - 1; ++j) issue(j);
    int in_block = 0;
    for (int j = 0; j < total; ++j) {
        cp_async_wait<S - 2>();  // this lane's copies of row j have landed
        const int r = gw + j * nwt;
        const unsigned char* st = ring + (j % S) * SB;
        const float rs = *reinterpret_cast<const float*>(st + NTEN * VPT * 512 + lane * 4);
        uint4 xv[VPT], dv[VPT], hv[RES ? VPT : 1];
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = lane + 32 * i;
            const uint4 z = make_uint4(0u, 0u, 0u, 0u);
            xv[i] = v < nvec ? *reinterpret_cast<const uint4*>(st + (0 * VPT + i) * 512 + lane * 16) : z;
            dv[i] = v < nvec ? *reinterpret_cast<const uint4*>(st + (1 * VPT + i) * 512 + lane * 16) : z;
            if constexpr (RES)
                hv[i] = v < nvec ? *reinterpret_cast<const uint4*>(st + (2 * VPT + i) * 512 + lane * 16) : z;
        }
        // pass 1: the row's sum of g * (-xh)
        const float2 nrs = make_float2(-rs, -rs);
        float2 d2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const uint32_t xw[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
            const uint32_t dw4[4] = {dv[i].x, dv[i].y, dv[i].z, dv[i].w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 nx = mul2(bf16x2_to_f2(xw[k]), nrs);
                const float2 gg = mul2(bf16x2_to_f2(dw4[k]), w2[i][k]);
                d2 = fma2(gg, nx, d2);
            }
        }
        const float dot = warp_sum(d2.x + d2.y);
        // pass 2: dx = rstd (g + nx c), c = -dot / H; the row's dw terms
        const float cr = -dot * invH;
        const float2 c2v = make_float2(cr, cr);
        const float2 rs2 = make_float2(rs, rs);
        uint16_t* dxrow = p.dx.ptr + row_offset(r, p.heads, p.dx.st, p.dx.sk);
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = lane + 32 * i;
            if (v >= nvec) continue;
            const uint32_t xw[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
            const uint32_t dw4[4] = {dv[i].x, dv[i].y, dv[i].z, dv[i].w};
            uint32_t hw[4] = {0u, 0u, 0u, 0u};
            if constexpr (RES) {
                hw[0] = hv[i].x; hw[1] = hv[i].y; hw[2] = hv[i].z; hw[3] = hv[i].w;
            }
            uint32_t out[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 d = bf16x2_to_f2(dw4[k]);
                const float2 nx = mul2(bf16x2_to_f2(xw[k]), nrs);
                const float2 gg = mul2(d, w2[i][k]);
                float2 o = mul2(fma2(nx, c2v, gg), rs2);
                if constexpr (RES) o = add2(o, bf16x2_to_f2(hw[k]));
                out[k] = pack2(o);
                s2[i][k] = fma2(d, nx, s2[i][k]);
            }
            st16(dxrow + 8 * v, make_uint4(out[0], out[1], out[2], out[3]));
        }
        if (++in_block == 8) {  // eight-row FP32 blocks go into the FP64 total
#pragma unroll
            for (int i = 0; i < VPT; ++i)
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    acc[i][2 * k] -= (double)s2[i][k].x;
                    acc[i][2 * k + 1] -= (double)s2[i][k].y;
                    s2[i][k] = make_float2(0.f, 0.f);
                }
            in_block = 0;
        }
        issue(j + S - 1);
    }
    cp_async_wait<0>();

#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int v = lane + 32 * i;
        if (v >= nvec) continue;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            tot[(size_t)warp * H + 8 * v + 2 * k] = acc[i][2 * k] - (double)s2[i][k].x;
            tot[(size_t)warp * H + 8 * v + 2 * k + 1] = acc[i][2 * k + 1] - (double)s2[i][k].y;
        }
    }
    __syncthreads();
    for (int col = threadIdx.x; col < H; col += blockDim.x) {
        double a = tot[col];
        for (int b = 1; b < nw; ++b) a += tot[(size_t)b * H + col];
        atomicAdd(p.acc + col, a);
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) last = (atomicAdd(p.ticket, 1u) == gridDim.x - 1) ? 1u : 0u;
    __syncthreads();
    if (last) {
        __threadfence();
        finish_dw(p, threadIdx.x, blockDim.x);
        if (threadIdx.x == 0) *p.ticket = 0u;
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
    const bool shard = p.seg_out != nullptr;
    const int nseg = shard ? p.n_seg_out : p.fold_segments;
    const int n = p.n_chunks;
    const int seg_len = p.seg_len;
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
        if (shard) {
            p.seg_out[(size_t)warp * p.H + col] = a;  // this shard's segment sums
        } else {
            seg[warp][lane] = a;
        }
    }
    if (shard) return;
    __syncthreads();
    if (warp == 0 && col < p.H) {
        double tot = seg[0][lane];
        for (int q = 1; q < nseg; ++q)
            if (q * seg_len < n) tot += seg[q][lane];
        store_dw(p, col, tot);
    }
}

// Final fold of a row-sharded deterministic backward: the table of every shard's segment
// sums, in segment order, folded left to right per column and rounded once.
__global__ void __launch_bounds__(256) fold_segments_kernel(const double* seg, int n_nonempty,
                                                            int H, float* dw, int accumulate) {
    const int col = blockIdx.x * blockDim.x + threadIdx.x;
    if (col >= H) return;
    double tot = __ldcg(seg + col);
    for (int q = 1; q < n_nonempty; ++q) tot += __ldcg(seg + (size_t)q * H + col);
    const float v = __double2float_rn(tot);
    dw[col] = accumulate ? __fadd_rn(dw[col], v) : v;
}

// ============================================================================================
// Small-row single kernel: row tasks (dx) and column tasks (dw, the full fixed order).
// ============================================================================================

constexpr int kSmallThreads = 512;
constexpr int kColStrip = 64;   // columns per column task
constexpr int kRowBatch = 8;    // rows loaded together by a column-task lane: one block of the
                                 // single-launch regime's order (short code: with a cold L2 the
                                 // instructions come from DRAM too)

template <int TPR, int VPT, bool RES, bool W32>
__global__ void __launch_bounds__(kSmallThreads, 2) bwd_small_kernel(const BwdParams p) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int H = p.H;
    // column tasks take the first block indices (they are the longer tasks, so they start
    // first); row tasks follow
    const int n_col_ctas = (H + kColStrip - 1) / kColStrip;
    if ((int)blockIdx.x >= n_col_ctas) {
        // ---- row task: TPR threads per row (TPR * VPT * 8 >= H), 256 / TPR rows per CTA.
        // The code stays short (VPT <= 4): when the L2 is cold the kernel's own instructions
        // come from DRAM, so its size is part of the latency.
        constexpr int RPC = kSmallThreads / TPR;
        constexpr int WPR = TPR / 32;
        __shared__ float red[RPC][WPR > 1 ? WPR : 1];
        const int rl = threadIdx.x / TPR;
        const int tr = threadIdx.x - rl * TPR;
        const int r = ((int)blockIdx.x - n_col_ctas) * RPC + rl;
        const bool rv = r < p.R;
        const int64_t ox = rv ? row_offset(r, p.heads, p.x.st, p.x.sk) : 0;
        const int64_t ody = rv ? row_offset(r, p.heads, p.dy.st, p.dy.sk) : 0;
        const float rs = rv ? __ldg(p.rstd + r) : 0.f;
        uint4 xv[VPT], dyv[VPT];
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = tr + TPR * i;
            const bool ok = rv && v < p.nvec;
            xv[i] = ok ? ld_stream16(p.x.ptr + ox + 8 * v) : make_uint4(0u, 0u, 0u, 0u);
            dyv[i] = ok ? ld_stream16(p.dy.ptr + ody + 8 * v) : make_uint4(0u, 0u, 0u, 0u);
        }
        float wf[VPT][8];
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = tr + TPR * i;
            if (v < p.nvec) {
                load_w8<W32>(p.w, 8 * v, wf[i]);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) wf[i][e] = 0.f;
            }
        }
        float d = 0.f;
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            float xf[8], df[8];
            unpack8(xv[i], xf);
            unpack8(dyv[i], df);
#pragma unroll
            for (int e = 0; e < 8; ++e)
                d = __fmaf_rn(__fmul_rn(df[e], wf[i][e]), __fmul_rn(xf[e], rs), d);
        }
        d = warp_sum(d);
        if constexpr (WPR > 1) {
            if (lane == 0) red[rl][warp - rl * WPR] = d;
            __syncthreads();
            d = 0.f;
#pragma unroll
            for (int w2 = 0; w2 < WPR; ++w2) d += red[rl][w2];
        }
        if (!rv) return;
        const float cr = __fdiv_rn(d, (float)H);
        const int64_t odx = row_offset(r, p.heads, p.dx.st, p.dx.sk);
        int64_t odh = 0;
        if constexpr (RES) odh = row_offset(r, p.heads, p.dh.st, p.dh.sk);
#pragma unroll
        for (int i = 0; i < VPT; ++i) {
            const int v = tr + TPR * i;
            if (v >= p.nvec) continue;
            float xf[8], df[8], out[8];
            unpack8(xv[i], xf);
            unpack8(dyv[i], df);
            float hf[8];
            if constexpr (RES) unpack8(ld_stream16(p.dh.ptr + odh + 8 * v), hf);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float xh = __fmul_rn(xf[e], rs);
                const float g = __fmul_rn(df[e], wf[i][e]);
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
    const int c0 = (int)blockIdx.x * kColStrip;
    const int j = c0 + 2 * lane;  // this lane's column pair
    const bool jok = j < H;
    const int B = p.block_rows;
    const int n_blocks = (p.R + B - 1) / B;
    const float2 m1 = make_float2(-1.f, -1.f);
    for (int b = warp; b < n_blocks; b += kSmallThreads / 32) {
        // TwoSum state (sum, compensation) of the lane's two columns, as packed pairs: every
        // packed operation rounds each lane like the scalar one, and the code is half as long
        float2 s2 = make_float2(0.f, 0.f), k2 = make_float2(0.f, 0.f);
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
                    // exact product p + e == dy * xh, then TwoSum of (s, p), per column
                    const float2 d = bf16x2_to_f2(dw2[u]);
                    const float2 xh = mul2(bf16x2_to_f2(xw[u]), make_float2(rs, rs));
                    const float2 pp = mul2(d, xh);
                    const float2 e = fma2(d, xh, mul2(pp, m1));
                    const float2 tt = add2(s2, pp);
                    const float2 z = sub2(tt, s2);
                    const float2 err = add2(sub2(s2, sub2(tt, z)), sub2(pp, z));
                    k2 = add2(k2, add2(err, e));
                    s2 = tt;
                }
            }
        }
        bp[(size_t)b * kColStrip + 2 * lane] = (double)s2.x + (double)k2.x;
        bp[(size_t)b * kColStrip + 2 * lane + 1] = (double)s2.y + (double)k2.y;
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
        store_dw(p, c0 + t, tot);
    }
}

// ============================================================================================
// host side
// ============================================================================================

namespace {


cudaError_t launch_fold(const BwdParams& p, cudaStream_t s);

// Shared memory one CTA of the staged kernel may take when MINB of them share an SM (228 KB
// per SM, 1 KB of it reserved per CTA).
constexpr size_t staged_budget(int minb) {
    return minb == 1 ? 220 * 1024 : minb == 2 ? 112 * 1024 : minb == 3 ? 74 * 1024 : 55 * 1024;
}

template <int ST, int VPT, int L, int P, bool DET, int NV, bool RES, bool W32, int MINB>
cudaError_t launch_large(const BwdParams& p, int grid_ctas, cudaStream_t s) {
    auto kern = bwd_staged_kernel<ST, VPT, L, P, DET, NV, RES, W32, MINB>;
    constexpr int NT = 32 + ST * L;
    constexpr int NTEN = RES ? 3 : 2;
    constexpr size_t kBudget = staged_budget(MINB);
    StagedCfg sc;
    sc.xch_rows = det_xch_rows(DET, L, p.block_rows);
    const size_t xch = (size_t)sc.xch_rows * p.nvec * 8 * sizeof(double);
    sc.xch_offset = kStagedHeader;
    sc.stage_offset = (int32_t)(kStagedHeader + ((xch + 127) & ~size_t(127)));
    sc.tensor_bytes = L * P * p.H * 2;
    sc.stage_bytes = NTEN * sc.tensor_bytes;
    int ns = (int)((kBudget - sc.stage_offset) / sc.stage_bytes);
    if (ns > kMaxStages) ns = kMaxStages;
    if (ns < 2) return cudaErrorInvalidConfiguration;
    if (!DET && (size_t)ns * sc.stage_bytes < (size_t)L * p.nvec * 8 * sizeof(double))
        return cudaErrorInvalidConfiguration;  // the slot totals must fit in the ring
    sc.n_stages = ns;
    const size_t smem = (size_t)sc.stage_offset + (size_t)ns * sc.stage_bytes;
    static SmemGrant granted;
    cudaError_t ge = grant_smem(granted, current_device(), kern, smem);
    if (ge != cudaSuccess) return ge;
    int grid = grid_ctas;
    if (grid <= 0) {
        const int64_t cap = (int64_t)device_sm_count() * MINB;
        int64_t need = DET ? p.n_chunks : ((int64_t)p.R + L * 8 - 1) / (L * 8);
        if (need < 1) need = 1;
        grid = (int)(need < cap ? need : cap);
    }
    RowMaps tm;
    const RowsIn views[3] = {p.x, p.dy, p.dh};
    make_row_maps(&tm, views, RES ? 3 : 2, p.heads, p.H, p.R, P);
    kern<<<grid, NT, smem, s>>>(p, sc, tm);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || !DET) return e;
    return launch_fold(p, s);
}

// Mid-sized blocked-FP32 backward of narrow rows: one warp per row, VPT vectors per lane, an
// S-stage cp.async ring per warp, 8-warp CTAs.
template <int VPT, int S, bool RES, bool W32>
cudaError_t launch_warp_bwd(const BwdParams& p, int grid_ctas, cudaStream_t s) {
    auto kern = bwd_warp_kernel<VPT, S, RES, W32>;
    constexpr int nw = kWarpBwdWarps;
    if (p.nvec > 32 * VPT) return cudaErrorInvalidConfiguration;
    const size_t ring = (size_t)nw * S * warp_stage_bytes<VPT, RES>();
    const size_t smem = (size_t)nw * p.H * sizeof(double) + ring;
    const size_t smem_max = (size_t)nw * 256 * VPT * sizeof(double) + ring;  // widest row
    // resident CTAs per SM at the widest row of this instantiation, per device
    static SmemGrant granted;
    static PerDevice<1> occ_cache;
    const int dev = current_device();
    cudaError_t e = grant_smem(granted, dev, kern, smem_max);
    if (e != cudaSuccess) return e;
    const int occ = resident_ctas(occ_cache, dev, 0, kern, nw * 32, smem_max, &e);
    if (occ < 0) return e;
    int grid = grid_ctas;
    if (grid <= 0) {
        int64_t need = ((int64_t)p.R + nw - 1) / nw;
        if (need < 1) need = 1;
        const int64_t cap = (int64_t)device_sm_count() * occ;
        grid = (int)(need < cap ? need : cap);
    }
    kern<<<grid, nw * 32, smem, s>>>(p);
    return cudaGetLastError();
}

template <bool RES, bool W32>
cudaError_t dispatch_warp_bwd(const BwdParams& p, int grid_ctas, cudaStream_t s) {
    constexpr int S = RES ? 6 : 8;
    if (p.nvec <= 32) return launch_warp_bwd<1, S, RES, W32>(p, grid_ctas, s);
    return launch_warp_bwd<2, S, RES, W32>(p, grid_ctas, s);
}

// fold kernel after a deterministic main kernel, programmatic dependent launch
cudaError_t launch_fold(const BwdParams& p, cudaStream_t s) {
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

// Rows of a slot per stage: 4 when two such stages fit beside the exchange area, else 2.
// The deterministic consumer gets the whole-width instantiation when the row is exactly
// ST*VPT vectors and a slot has at least two warps (measured 4-16 % faster at H 1536-6144;
// with fewer threads per row the compiler hoists a whole tile's loads once the offsets are
// constant, and spills; the blocked-FP32 consumer measured slower with it).
template <int ST, int VPT, int L, int P, bool DET, bool RES, bool W32, int MINB>
cudaError_t launch_large_nv(const BwdParams& p, int grid_ctas, cudaStream_t s) {
    if constexpr (DET && ST >= 64) {
        if (p.nvec == ST * VPT)
            return launch_large<ST, VPT, L, P, DET, ST * VPT, RES, W32, MINB>(p, grid_ctas, s);
    }
    return launch_large<ST, VPT, L, P, DET, 0, RES, W32, MINB>(p, grid_ctas, s);
}

// MINB: CTAs of the layout that share an SM (each with its own producer and stage ring).
template <int ST, int VPT, int L, bool DET, bool RES, bool W32, int MINB = 1>
cudaError_t launch_large_p(const BwdParams& p, int grid_ctas, cudaStream_t s) {
    constexpr size_t kRoom = staged_budget(MINB) - kStagedHeader;
    const size_t xch = (size_t)det_xch_rows(DET, L, p.block_rows) * p.nvec * 8 * sizeof(double);
    const size_t row = (size_t)(RES ? 3 : 2) * L * p.H * 2;
    if (2 * 4 * row + xch + 128 <= kRoom)
        return launch_large_nv<ST, VPT, L, 4, DET, RES, W32, MINB>(p, grid_ctas, s);
    return launch_large_nv<ST, VPT, L, 2, DET, RES, W32, MINB>(p, grid_ctas, s);
}

// Slot layout per width: ST threads per slot, VPT vectors per thread, L slots per CTA.  L is
// also the block count of a deterministic chunk and depends on the width only (it must match
// bwd_slots_for_width); ST and VPT are free and were measured per width and mode: narrow rows
// share a warp between rows, and the deterministic mode, which carries a TwoSum state per
// column, runs best with more threads and fewer columns per thread.
constexpr int kThinDetRows = 131072;

template <bool DET, bool RES, bool W32>
cudaError_t dispatch_large(const BwdParams& p, int grid_ctas, cudaStream_t s) {
    const int nv = p.nvec;
    if constexpr (!DET) {
        if (nv <= 64 && (int64_t)p.R * p.H < kWarpBwdMaxElems)
            return dispatch_warp_bwd<RES, W32>(p, grid_ctas, s);
    }
    // H <= 256, both modes: half-warp slots, 8 per CTA, two CTAs per SM, each with its own
    // producer and ring (measured against one CTA of 16 slots: deterministic [1024,24,256]
    // 21.0 vs 24.5 us, [16384,4,256] 34.3 vs 38.5 us; blocked FP32 H 256 x 1M 278 vs 295 us;
    // within 2 % either way at [16384,24,256]; slower at H 512, which keeps one CTA).  The
    // deterministic mode takes three CTAs per SM from 131072 rows (128 registers, no spill:
    // [16384,24,256] 136 vs 154 us, H 256 x 1M 319 vs 343 us; 4 % slower at 65536 rows)
    if constexpr (DET) {
        if (nv <= 32 && p.R >= kThinDetRows)
            return launch_large_p<16, 2, 8, DET, RES, W32, 3>(p, grid_ctas, s);
    }
    if (nv <= 32) return launch_large_p<16, 2, 8, DET, RES, W32, 2>(p, grid_ctas, s);
    if constexpr (DET) {
        // thinner slots at H 512 from 131072 rows: twice the consumer warps (H 512 x 131072
        // 100 vs 105 us; slower at fewer rows); same L, same order
        if (p.R >= kThinDetRows && nv <= 64)
            return launch_large_p<64, 1, 8, DET, RES, W32>(p, grid_ctas, s);
    }
    if (nv <= 64) return launch_large_p<32, 2, 8, DET, RES, W32>(p, grid_ctas, s);
    if (nv <= 128) return launch_large_p<64, 2, 4, DET, RES, W32>(p, grid_ctas, s);
    if constexpr (DET) {
        // H 2048: one slot of 128 threads with two vectors each per CTA, three CTAs per SM,
        // each with its own producer and ring, so no slot waits for another to release a
        // stage (the order's L is 1 at this width; 128 registers).  Measured at 65537 rows:
        // 157 us against 178 with 256 x 1 at two CTAs per SM; at four CTAs per SM the
        // registers spill.  At H 1536 (L 4) neither 64 x 3 x 4 (spills at two CTAs per SM,
        // slower at one) nor 192 x 1 at two CTAs per SM beats 96 x 2 x 4.
        if (nv <= 192) return launch_large_p<96, 2, 4, DET, RES, W32>(p, grid_ctas, s);
        if (nv <= 256) return launch_large_p<128, 2, 1, DET, RES, W32, 3>(p, grid_ctas, s);
    }
    // blocked FP32 (measured: H 1536 x 65537 112 vs 116 us with 192 x 1 against 96 x 2; H 2048
    // x 65537 143 vs 155 us with 128 x 2 against 256 x 1)
    if (nv <= 192) return launch_large_p<192, 1, 2, DET, RES, W32>(p, grid_ctas, s);
    if (nv <= 256) return launch_large_p<128, 2, 2, DET, RES, W32>(p, grid_ctas, s);
    if (nv <= 384) return launch_large_p<128, 3, 2, DET, RES, W32>(p, grid_ctas, s);
    if (nv <= 512) return launch_large_p<512, 1, 1, DET, RES, W32>(p, grid_ctas, s);
    if (nv <= 640) return launch_large_p<640, 1, 1, DET, RES, W32>(p, grid_ctas, s);
    if (nv <= 768) {
        if constexpr (DET) return launch_large_p<384, 2, 1, DET, RES, W32>(p, grid_ctas, s);
        else return launch_large_p<256, 3, 1, DET, RES, W32>(p, grid_ctas, s);
    }
    if constexpr (DET) return launch_large_p<512, 2, 1, DET, RES, W32>(p, grid_ctas, s);
    else return launch_large_p<256, 4, 1, DET, RES, W32>(p, grid_ctas, s);
}

template <int TPR, int VPT, bool RES, bool W32>
cudaError_t launch_small_t(const BwdParams& p, cudaStream_t s) {
    auto kern = bwd_small_kernel<TPR, VPT, RES, W32>;
    constexpr int RPC = kSmallThreads / TPR;
    const int n_row_ctas = (p.R + RPC - 1) / RPC;
    const int n_col_ctas = (p.H + kColStrip - 1) / kColStrip;
    const int n_blocks = (p.R + p.block_rows - 1) / p.block_rows;
    const size_t smem = (size_t)n_blocks * kColStrip * sizeof(double);
    static SmemGrant granted;
    if (smem > 48 * 1024) {
        cudaError_t e = grant_smem(granted, current_device(), kern, smem);
        if (e != cudaSuccess) return e;
    }
    kern<<<n_row_ctas + n_col_ctas, kSmallThreads, smem, s>>>(p);
    return cudaGetLastError();
}

// Threads per row: one warp up to 256 columns, then up to 256 threads, then more vectors
// per thread.
template <bool RES, bool W32>
cudaError_t dispatch_small(const BwdParams& p, cudaStream_t s) {
    const int nv = p.nvec;
    if (nv <= 32) return launch_small_t<32, 1, RES, W32>(p, s);
    if (nv <= 64) return launch_small_t<64, 1, RES, W32>(p, s);
    if (nv <= 128) return launch_small_t<128, 1, RES, W32>(p, s);
    if (nv <= 256) return launch_small_t<256, 1, RES, W32>(p, s);
    if (nv <= 512) return launch_small_t<256, 2, RES, W32>(p, s);
    if (nv <= 768) return launch_small_t<256, 3, RES, W32>(p, s);
    return launch_small_t<256, 4, RES, W32>(p, s);
}

}  // namespace

int bwd_slots_for_width(int H) {
    const int nv = H / 8;
    if (nv <= 32) return 8;
    if (nv <= 64) return 8;
    if (nv <= 192) return 4;
    if (nv <= 256) return 1;
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

cudaError_t launch_fold_segments(const double* seg, int n_nonempty, int H, float* dw,
                                 int accumulate, cudaStream_t s) {
    fold_segments_kernel<<<(H + 255) / 256, 256, 0, s>>>(seg, n_nonempty, H, dw, accumulate);
    return cudaGetLastError();
}

cudaError_t launch_bwd_nondet(const BwdParams& p, bool res, bool w32, int grid_ctas,
                              cudaStream_t s) {
    if (res) return w32 ? dispatch_large<false, true, true>(p, grid_ctas, s)
                        : dispatch_large<false, true, false>(p, grid_ctas, s);
    return w32 ? dispatch_large<false, false, true>(p, grid_ctas, s)
               : dispatch_large<false, false, false>(p, grid_ctas, s);
}

}  // namespace rmsk
