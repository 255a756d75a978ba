// Internal declarations shared by the kernels and the C-ABI layer of librmsnorm_train.
#pragma once

#include <cuda.h>  // CUtensorMap and its enums (types only; the encoder is fetched at run time)
#include <cuda_runtime.h>
#include <stdint.h>

#include "launch_cache.h"
#include "rmsnorm_train.h"

namespace rmsk {

// A [T, heads, H] row view: row (t, k) starts at element t*st + k*sk.
struct RowsIn {
    const uint16_t* ptr;
    int64_t st, sk;
};
struct RowsOut {
    uint16_t* ptr;
    int64_t st, sk;
};

struct FwdParams {
    int32_t R;       // rows = T * heads
    int32_t heads;
    int32_t H;
    int32_t nvec;    // H / 8 (16-byte vectors per row)
    RowsIn x;
    RowsIn res;      // residual form only
    RowsOut h;       // residual form only
    RowsOut y;
    const void* w;
    float* rstd;
    float eps;
    // rows ahead of the current one whose inputs are prefetched into L2 (0: none)
    int32_t prefetch;
};

struct BwdParams {
    int32_t R;
    int32_t heads;
    int32_t H;
    int32_t nvec;
    RowsIn x;        // h in the residual form
    RowsIn dy;
    RowsIn dh;       // residual form only
    RowsOut dx;      // grad_h in the residual form
    const void* w;
    const float* rstd;
    float* dw;
    // workspace pieces
    unsigned* status;    // device error word
    unsigned* ticket;    // non-deterministic grid combine
    double* acc;         // [H] FP64, zero between calls
    double* part;        // [n_chunks, H] FP64 chunk partials (deterministic)
    // deterministic order
    int32_t block_rows;
    int32_t blocks_per_chunk;
    int32_t fold_segments;
    int32_t n_chunks;        // chunks of this call's rows
    int32_t seg_len;         // chunks per fold segment (of the whole problem's plan)
    // Row-sharded deterministic calls: when non-null the fold kernel writes the FP64 sums
    // of this shard's n_seg_out segments ([n_seg_out][H]; 0 for an empty segment) instead
    // of folding them into dw.
    double* seg_out;
    int32_t n_seg_out;
    // limit of every device-side wait, in SM clock cycles
    int64_t wait_cycles;
    // 0: dw = the call's sum; 1: dw = FP32(dw + FP32(the call's sum)), the FP32 sum of the
    // previous dw and the value the overwrite mode returns
    int32_t accumulate;
};

// TMA descriptors of up to three row tensors (x / dy / dh, or x / residual); use[i] != 0
// when tensor i has equally spaced rows of H <= 256 and its descriptor is valid.
struct alignas(64) RowMaps {
    CUtensorMap map[3];
    int32_t use[3];
};

// device status bits
constexpr unsigned kStatusTimeout = 1u;
// default limit of a device-side wait (about two seconds at 2 GHz)
constexpr int64_t kDefaultWaitCycles = 4000000000LL;

// Raises `kern`'s dynamic shared-memory limit on the current device `dev` to at least
// `bytes`, once per device (see SmemGrant).
template <typename K>
cudaError_t grant_smem(SmemGrant& g, int dev, K kern, size_t bytes) {
    return static_cast<cudaError_t>(g.grant(dev, (int)bytes, [&](int b) {
        return (int)cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, b);
    }));
}

// Resident CTAs per SM of `kern` at (threads, smem) on device `dev`, cached per device under
// `key` (at least 1; -1 when the occupancy query fails, with the error in *err).
template <int N, typename K>
int resident_ctas(PerDevice<N>& cache, int dev, int key, K kern, int threads, size_t smem,
                  cudaError_t* err) {
    return cache.get(dev, key, [&]() {
        int o = 0;
        *err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, kern, threads, smem);
        if (*err != cudaSuccess) return -1;
        return o > 0 ? o : 1;
    });
}

// ---- host-side launchers (defined in fwd.cu / bwd.cu) -------------------------------------

cudaError_t launch_fwd(const FwdParams& p, bool residual, bool w32, cudaStream_t s);
cudaError_t launch_bwd_small(const BwdParams& p, bool residual, bool w32, cudaStream_t s);
cudaError_t launch_bwd_det(const BwdParams& p, bool residual, bool w32, int grid_ctas,
                           cudaStream_t s);
cudaError_t launch_bwd_nondet(const BwdParams& p, bool residual, bool w32, int grid_ctas,
                              cudaStream_t s);
// Folds a table of FP64 segment sums seg[n_seg][H] (the first n_nonempty non-empty) left to
// right per column and rounds once to FP32 into dw (added to dw when accumulate != 0).
cudaError_t launch_fold_segments(const double* seg, int n_nonempty, int H, float* dw,
                                 int accumulate, cudaStream_t s);

// Rows processed together by one CTA of the large backward kernels for this width
// (the blocks of one deterministic chunk).  Also the chunk's block count.
int bwd_slots_for_width(int H);
// The current device (cudaGetDevice; -1 on error) and its SM count (cached per device).
int current_device();
int device_sm_count();
// Fills `maps` for the first n views (box of box_rows rows x H); tensors that cannot use a
// descriptor get use = 0 and keep the bulk-copy path.
void make_row_maps(RowMaps* maps, const RowsIn* views, int n, int heads, int H, int64_t rows,
                   int box_rows);
// Records `msg` as this thread's rms_last_error() text and returns `code`.
int set_error(int code, const char* msg);

// Called by the backward entry after every host-side check of a call has passed and just
// before its first launch; a non-zero return ends the call with that code.
typedef int (*PreLaunchFn)(void* ctx, cudaStream_t s);

// The backward behind rms_train_bwd / rms_residual_train_bwd (dh == nullptr for the plain
// form), with an optional hook run right before the launches.
int bwd_entry(rms_shape shape, rms_rows x, const void* w, int w_dtype, const float* rstd,
              rms_rows dy, const rms_rows* dh, rms_rows dx, float* dw, int deterministic,
              void* ws, size_t ws_bytes, int grid_ctas, void* stream, PreLaunchFn hook,
              void* hook_ctx);

}  // namespace rmsk

// ---- device helpers ------------------------------------------------------------------------
#ifdef __CUDACC__
namespace rmsk {

__device__ __forceinline__ float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// two FP32 -> packed BF16x2, round to nearest even (low half = a)
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
    return r;
}

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
    f[0] = bf16lo(v.x); f[1] = bf16hi(v.x);
    f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
    f[4] = bf16lo(v.z); f[5] = bf16hi(v.z);
    f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
    uint4 v;
    v.x = pack_bf16x2(f[0], f[1]);
    v.y = pack_bf16x2(f[2], f[3]);
    v.z = pack_bf16x2(f[4], f[5]);
    v.w = pack_bf16x2(f[6], f[7]);
    return v;
}

// 16-byte streaming load of data read once (no L1 allocation).
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(p));
    return v;
}

// 16-byte load through L1 (small, reused data: the weight).
__device__ __forceinline__ uint4 ld_cached16(const void* p) {
    return __ldg(reinterpret_cast<const uint4*>(p));
}

__device__ __forceinline__ void st16(void* p, const uint4& v) {
    *reinterpret_cast<uint4*>(p) = v;
}

// 8 weights as FP32 from a BF16 or FP32 weight vector, element offset e (multiple of 8).
template <bool W32>
__device__ __forceinline__ void load_w8(const void* w, int e, float (&f)[8]) {
    if constexpr (W32) {
        const float* wf = static_cast<const float*>(w) + e;
        uint4 a = ld_cached16(wf), b = ld_cached16(wf + 4);
        f[0] = __uint_as_float(a.x); f[1] = __uint_as_float(a.y);
        f[2] = __uint_as_float(a.z); f[3] = __uint_as_float(a.w);
        f[4] = __uint_as_float(b.x); f[5] = __uint_as_float(b.y);
        f[6] = __uint_as_float(b.z); f[7] = __uint_as_float(b.w);
    } else {
        uint4 a = ld_cached16(static_cast<const uint16_t*>(w) + e);
        unpack8(a, f);
    }
}

// ---- packed FP32 pairs (sm_100 f32x2 instructions; each lane rounds like the scalar op) ----

__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t u) {
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
// a - b, exactly one rounding (fma with -1 is exact before the rounding)
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
    return __ffma2_rn(b, make_float2(-1.f, -1.f), a);
}
__device__ __forceinline__ uint32_t pack2(float2 v) { return pack_bf16x2(v.x, v.y); }

// The one FP32 rounding of a dw column's FP64 total, stored or added to the previous dw.
__device__ __forceinline__ void store_dw(const BwdParams& p, int col, double total) {
    const float v = __double2float_rn(total);
    p.dw[col] = p.accumulate ? __fadd_rn(p.dw[col], v) : v;
}

__device__ __forceinline__ int64_t row_offset(int32_t r, int32_t heads, int64_t st,
                                              int64_t sk) {
    if (heads == 1) return (int64_t)r * st;
    if (st == (int64_t)heads * sk) return (int64_t)r * sk;  // equally spaced rows: no division
    const int32_t t = r / heads;
    const int32_t k = r - t * heads;
    return (int64_t)t * st + (int64_t)k * sk;
}

// True when consecutive rows of the view follow each other in memory (row r + 1 starts
// where row r ends), so a run of rows is one contiguous byte range.
__device__ __forceinline__ bool rows_contiguous(const RowsIn& v, int32_t heads, int32_t H) {
    return heads == 1 ? v.st == H : (v.sk == H && v.st == (int64_t)heads * H);
}

// Sum over each group of G consecutive lanes (G a power of two, at most 32); every lane
// receives its group's sum.
template <int G>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    return v;
}

__device__ __forceinline__ float warp_sum(float v) { return group_sum<32>(v); }

// ---- per-thread asynchronous copies (cp.async): a thread waits for its own copies only -------
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---- shared-memory barriers and bulk copies (sm_90+ PTX) -----------------------------------

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// make barrier initialisation visible to the bulk-copy (async) proxy
__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}

// Non-blocking probe of the phase of `parity`.
__device__ __forceinline__ bool mbar_probe(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}

// Waits for the phase of `parity` to complete; gives up after `limit` SM cycles and
// returns false.  Never waits forever.  A limit of 0 is a single non-blocking probe
// (try_wait itself may suspend the thread for a while before returning).
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, int64_t limit) {
    if (limit <= 0) return mbar_probe(bar, parity);
    if (mbar_test(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_test(bar, parity)) return true;
        if (clock64() - t0 > limit) return false;
    }
}

// 2-D tiled TMA load of rows [row0, row0 + box rows) of a row tensor (box = H x rows) into
// shared memory, completion counted on `bar`.  x is always 0 (16-byte aligned); rows past
// the tensor's end are filled with zeros and still counted.
__device__ __forceinline__ void tma_load_rows(uint32_t dst, const CUtensorMap* map, int row0,
                                              uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(row0), "r"(bar)
        : "memory");
}

// Bulk prefetch of [src, src + bytes) into L2 (no destination, nothing to wait for); src
// and bytes must be multiples of 16.
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Bulk copy global -> shared (this CTA), completion counted in bytes on `bar`.
// dst, src and bytes must be multiples of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

}  // namespace rmsk
#endif
