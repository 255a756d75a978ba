// C ABI of librmsnorm_train: argument checks, workspace layout, program choice.
// The declarations and their contract are in include/rmsnorm_train.h.
#include <atomic>
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "common.cuh"
#include "rmsnorm_train.h"

namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

int ok() {
    g_err.clear();
    return RMS_OK;
}

int cuda_fail(cudaError_t e, const char* what) {
    return fail(RMS_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr int kMaxH = 8192;
constexpr int kFoldSegments = 16;
constexpr size_t kWsHeader = 256;  // status word, ticket
// The FP64 accumulator of the non-deterministic combine is kept zero between calls.  It
// is reserved for the widest row so that the deterministic chunk partials, which follow
// it, never land on it whatever the H of the call that wrote them.
constexpr size_t kAccBytes = (size_t)kMaxH * 8;

// process-wide settings (rms_set_small_rows_limit, rms_set_wait_limit_cycles)
std::atomic<int64_t> g_small_rows_override{-1};
std::atomic<int64_t> g_wait_cycles{rmsk::kDefaultWaitCycles};
std::atomic<int> g_prefetch{-1};  // -1: the library's choice

struct Span {
    uintptr_t lo, hi;  // [lo, hi)
    const char* name;
};

bool overlap(const Span& a, const Span& b) {
    return a.lo < a.hi && b.lo < b.hi && a.lo < b.hi && b.lo < a.hi;
}

int check_shape(const rms_shape& s) {
    if (s.T < 0) return fail(RMS_EINVAL, "T must be >= 0 (got %lld)", (long long)s.T);
    if (s.heads < 1) return fail(RMS_EINVAL, "heads must be >= 1 (got %d)", s.heads);
    if (s.H < 8 || s.H > kMaxH || s.H % 8 != 0)
        return fail(RMS_EINVAL, "H must be a multiple of 8 in [8, %d] (got %d)", kMaxH, s.H);
    if (s.T > 0 && (int64_t)s.T * s.heads >= (int64_t(1) << 31))
        return fail(RMS_EINVAL, "T*heads must be < 2^31");
    return RMS_OK;
}

// Checks a row view; appends its byte span.  `out` marks views that are written.
int check_rows(const rms_shape& s, const rms_rows& v, const char* name, bool out, Span* span) {
    if (!v.ptr) return fail(RMS_EINVAL, "%s is null", name);
    if (reinterpret_cast<uintptr_t>(v.ptr) % 16)
        return fail(RMS_EALIGN, "%s must be 16-byte aligned", name);
    const int64_t sk = s.heads > 1 ? v.sk : 0;
    if (v.st < 0 || sk < 0) return fail(RMS_EINVAL, "%s strides must be >= 0", name);
    if (v.st % 8 || sk % 8)
        return fail(RMS_EALIGN, "%s strides must be multiples of 8 elements", name);
    if (out) {
        if (s.heads > 1 && sk < s.H)
            return fail(RMS_EINVAL, "%s: head stride %lld makes output rows overlap", name,
                        (long long)sk);
        if (s.T > 1 && v.st < (int64_t)(s.heads - 1) * sk + s.H)
            return fail(RMS_EINVAL, "%s: token stride %lld makes output rows overlap", name,
                        (long long)v.st);
    }
    const int64_t n = (s.T - 1) * v.st + (int64_t)(s.heads - 1) * sk + s.H;
    span->lo = reinterpret_cast<uintptr_t>(v.ptr);
    span->hi = span->lo + (uintptr_t)n * 2;
    span->name = name;
    return RMS_OK;
}

int check_aliases(const Span* in, int nin, const Span* out, int nout) {
    for (int i = 0; i < nout; ++i) {
        for (int j = 0; j < nin; ++j)
            if (overlap(out[i], in[j]))
                return fail(RMS_EALIAS, "output %s overlaps input %s", out[i].name, in[j].name);
        for (int j = i + 1; j < nout; ++j)
            if (overlap(out[i], out[j]))
                return fail(RMS_EALIAS, "output %s overlaps output %s", out[i].name,
                            out[j].name);
    }
    return RMS_OK;
}

Span span_of(const void* p, size_t bytes, const char* name) {
    Span s;
    s.lo = reinterpret_cast<uintptr_t>(p);
    s.hi = s.lo + bytes;
    s.name = name;
    return s;
}

rmsk::RowsIn in_of(const rms_shape& s, const rms_rows& v) {
    return {static_cast<const uint16_t*>(v.ptr), v.st, s.heads > 1 ? v.sk : 0};
}
rmsk::RowsOut out_of(const rms_shape& s, const rms_rows& v) {
    return {static_cast<uint16_t*>(v.ptr), v.st, s.heads > 1 ? v.sk : 0};
}

// ---- the deterministic order and the program choice --------------------------------------

// Rows per block of the deterministic order: in the single-launch regime 8 up to 128 rows
// (at most 16 blocks: each warp of a column task sums one block after one round of loads;
// measured 1-1.5 us faster at T 32-87) and 16 up to 2048 rows (8-row blocks there give a warp
// two blocks and measured slower at T 227); otherwise the largest power of two in [8, 64]
// that still cuts the rows into at least kMinChunks chunks of L blocks (one per SM of a
// B200), so mid-sized problems keep every SM busy.  A function of (R, L) -- that is, of the
// row count and the width -- and of nothing else.
constexpr int64_t kMinChunks = 148;

int32_t det_block_rows(int64_t R, int L) {
    if (R <= 128) return 8;
    if (R <= 2048) return 16;
    int32_t B = 64;
    while (B > 8 && (R + (int64_t)B * L - 1) / ((int64_t)B * L) < kMinChunks) B /= 2;
    return B;
}

int64_t default_small_rows(int H) {
    // single-launch program up to about 2^20 elements (and its shared-memory bound)
    int64_t lim = (int64_t(1) << 20) / H;
    if (lim > 2048) lim = 2048;
    if (lim < 64) lim = 64;
    return lim;
}

// L2 prefetch of rows ahead (the pages' mid-size forward prefetch, PR #8656 introduction):
// rows ahead of the current one that the forward's one-CTA-per-row kernel (H > 1024) warms
// in L2.  Measured on B200: one row ahead gains 2-4 % below 32768 rows (H 6144 x 4096:
// 20.2 -> 19.4 us; residual H 6144 x 4096: 36.3 -> 35.7 us; H 4096 x 16384: 47.0 -> 46.3 us)
// and costs 3-8 % at 65537 rows and more, where every CTA walks hundreds of rows and the
// extra requests only compete with the loads; two rows ahead is slower than one.  The same
// prefetch in the backward's bulk-copy producer (the tile one ring ahead) cost 2-25 % and is
// not built.
constexpr int64_t kFwdPrefetchMaxRows = 32768;

int fwd_prefetch(int64_t R, int H) {
    const int v = g_prefetch.load();
    if (v >= 0) return v;
    return (H > 1024 && R < kFwdPrefetchMaxRows) ? 1 : 0;
}

bool use_small(int64_t R, int H) {
    const int64_t ov = g_small_rows_override.load();
    const int64_t lim = ov >= 0 ? ov : default_small_rows(H);
    return R <= lim && R <= 2048;
}

struct Plan {
    int32_t B, L, S, n_chunks;
    int32_t seg_len;  // chunks per fold segment
};

Plan det_plan(int64_t R, int H) {
    Plan p;
    p.L = rmsk::bwd_slots_for_width(H);
    p.B = det_block_rows(R, p.L);
    p.S = kFoldSegments;
    const int64_t ch = (int64_t)p.B * p.L;
    p.n_chunks = (int32_t)((R + ch - 1) / ch);
    p.seg_len = (p.n_chunks + p.S - 1) / p.S;
    return p;
}

// Rows of one rank of a row-sharded deterministic backward: the rank owns 16 / world whole
// fold segments of the plan of all T rows, so its rows are whole chunks and the folds of
// its segments are exactly those of the single-GPU order.
struct ShardPlan {
    int64_t row_begin, row_end;
    int32_t n_seg;          // segments of the rank (16 / world)
    int32_t n_chunks;       // chunks of the rank's rows
    size_t ws_bytes;
};

int shard_plan(const rms_shape& s, int rank, int world, ShardPlan* out) {
    int rc = check_shape(s);
    if (rc) return rc;
    if (s.heads != 1)
        return fail(RMS_EINVAL, "row sharding takes [T, H] rows (heads must be 1, got %d)",
                    s.heads);
    if (world < 1 || world > kFoldSegments || kFoldSegments % world)
        return fail(RMS_EINVAL, "world must divide %d (got %d)", kFoldSegments, world);
    if (rank < 0 || rank >= world)
        return fail(RMS_EINVAL, "rank must be in [0, %d) (got %d)", world, rank);
    const Plan pl = det_plan(s.T, s.H);
    const int per = kFoldSegments / world;
    const int64_t c0 = std::min<int64_t>(pl.n_chunks, (int64_t)rank * per * pl.seg_len);
    const int64_t c1 = std::min<int64_t>(pl.n_chunks, (int64_t)(rank + 1) * per * pl.seg_len);
    const int64_t ch = (int64_t)pl.B * pl.L;
    out->row_begin = std::min<int64_t>(s.T, c0 * ch);
    out->row_end = std::min<int64_t>(s.T, c1 * ch);
    out->n_seg = per;
    out->n_chunks = (int32_t)(c1 - c0);
    out->ws_bytes = kWsHeader + kAccBytes + (size_t)out->n_chunks * s.H * 8;
    return RMS_OK;
}

size_t ws_bytes(const rms_shape& s, int det) {
    const int64_t R = s.T * s.heads;
    size_t b = kWsHeader + kAccBytes;
    if (det && !use_small(R, s.H)) b += (size_t)det_plan(R, s.H).n_chunks * s.H * 8;
    return b;
}

// The workspace: present, 256-byte aligned, at least `need` bytes, apart from every input
// and output.
int check_workspace(void* ws, size_t ws_size, size_t need, const Span* ins, int nin,
                    const Span* outs, int nout) {
    if (!ws) return fail(RMS_EWORKSPACE, "workspace is null (needs %zu bytes)", need);
    if (reinterpret_cast<uintptr_t>(ws) % 256)
        return fail(RMS_EALIGN, "workspace must be 256-byte aligned");
    if (ws_size < need)
        return fail(RMS_EWORKSPACE, "workspace has %zu bytes, needs %zu", ws_size, need);
    const Span wsp = span_of(ws, need, "workspace");
    for (int i = 0; i < nin; ++i)
        if (overlap(wsp, ins[i])) return fail(RMS_EALIAS, "workspace overlaps %s", ins[i].name);
    for (int i = 0; i < nout; ++i)
        if (overlap(wsp, outs[i])) return fail(RMS_EALIAS, "workspace overlaps %s", outs[i].name);
    return RMS_OK;
}

int bwd_common(rms_shape shape, rms_rows x, const void* w, int w_dtype, const float* rstd,
               rms_rows dy, const rms_rows* dh, rms_rows dx, float* dw, int deterministic,
               void* ws, size_t ws_size, int grid_ctas, void* stream, int accumulate = 0,
               rmsk::PreLaunchFn hook = nullptr, void* hook_ctx = nullptr) {
    int rc = check_shape(shape);
    if (rc) return rc;
    if (w_dtype != RMS_BF16 && w_dtype != RMS_FP32)
        return fail(RMS_EDTYPE, "w_dtype must be RMS_BF16 or RMS_FP32 (got %d)", w_dtype);
    if (grid_ctas < 0 || grid_ctas > 65535)
        return fail(RMS_EINVAL, "grid_ctas must be in [0, 65535] (got %d)", grid_ctas);
    if (!w || !dw) return fail(RMS_EINVAL, "w and dw must not be null");
    if (reinterpret_cast<uintptr_t>(w) % 16 || reinterpret_cast<uintptr_t>(dw) % 16)
        return fail(RMS_EALIGN, "w and dw must be 16-byte aligned");
    const int64_t R = shape.T * shape.heads;
    const int H = shape.H;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t wb = (size_t)H * (w_dtype == RMS_FP32 ? 4 : 2);
    if (R == 0) {
        Span ins[1] = {span_of(w, wb, "w")};
        Span outs[1] = {span_of(dw, (size_t)H * 4, "dw")};
        if ((rc = check_aliases(ins, 1, outs, 1))) return rc;
        if (accumulate) return ok();  // adding an empty sum leaves dw as it is
        cudaError_t e = cudaMemsetAsync(dw, 0, (size_t)H * 4, st);
        return e == cudaSuccess ? ok() : cuda_fail(e, "cudaMemsetAsync(dw)");
    }
    if (!rstd) return fail(RMS_EINVAL, "rstd is null");
    if (reinterpret_cast<uintptr_t>(rstd) % 4) return fail(RMS_EALIGN, "rstd must be 4-byte aligned");
    Span ins[5], outs[2];
    int nin = 0;
    if ((rc = check_rows(shape, x, dh ? "h" : "x", false, &ins[nin++]))) return rc;
    if ((rc = check_rows(shape, dy, "dy", false, &ins[nin++]))) return rc;
    if (dh && (rc = check_rows(shape, *dh, "dh", false, &ins[nin++]))) return rc;
    ins[nin++] = span_of(w, wb, "w");
    ins[nin++] = span_of(rstd, (size_t)R * 4, "rstd");
    if ((rc = check_rows(shape, dx, dh ? "grad_h" : "dx", true, &outs[0]))) return rc;
    outs[1] = span_of(dw, (size_t)H * 4, "dw");
    if ((rc = check_aliases(ins, nin, outs, 2))) return rc;
    if ((rc = check_workspace(ws, ws_size, ws_bytes(shape, deterministic), ins, nin, outs, 2)))
        return rc;

    rmsk::BwdParams p = {};
    p.R = (int32_t)R;
    p.heads = shape.heads;
    p.H = H;
    p.nvec = H / 8;
    p.x = in_of(shape, x);
    p.dy = in_of(shape, dy);
    if (dh) p.dh = in_of(shape, *dh);
    p.dx = out_of(shape, dx);
    p.w = w;
    p.rstd = rstd;
    p.dw = dw;
    unsigned char* base = static_cast<unsigned char*>(ws);
    p.status = reinterpret_cast<unsigned*>(base);
    p.ticket = reinterpret_cast<unsigned*>(base + 4);
    p.acc = reinterpret_cast<double*>(base + kWsHeader);
    p.part = reinterpret_cast<double*>(base + kWsHeader + kAccBytes);
    const Plan plan = det_plan(R, H);
    p.block_rows = plan.B;
    p.blocks_per_chunk = plan.L;
    p.fold_segments = plan.S;
    p.n_chunks = plan.n_chunks;
    p.seg_len = plan.seg_len;
    p.wait_cycles = g_wait_cycles.load();
    p.accumulate = accumulate ? 1 : 0;
    const bool res = dh != nullptr;
    const bool w32 = w_dtype == RMS_FP32;
    if (hook && (rc = hook(hook_ctx, st))) return rc;
    cudaError_t e;
    if (use_small(R, H)) {
        e = rmsk::launch_bwd_small(p, res, w32, st);
    } else if (deterministic) {
        e = rmsk::launch_bwd_det(p, res, w32, grid_ctas, st);
    } else {
        e = rmsk::launch_bwd_nondet(p, res, w32, grid_ctas, st);
    }
    if (e != cudaSuccess) return cuda_fail(e, "backward launch");
    return ok();
}

int shard_common(rms_shape shape, int rank, int world, rms_rows x, const void* w, int w_dtype,
                 const float* rstd, rms_rows dy, rms_rows dh, rms_rows dx, double* seg_out,
                 void* ws, size_t ws_size, int grid_ctas, void* stream) {
    ShardPlan sp;
    int rc = shard_plan(shape, rank, world, &sp);
    if (rc) return rc;
    if (w_dtype != RMS_BF16 && w_dtype != RMS_FP32)
        return fail(RMS_EDTYPE, "w_dtype must be RMS_BF16 or RMS_FP32 (got %d)", w_dtype);
    if (grid_ctas < 0 || grid_ctas > 65535)
        return fail(RMS_EINVAL, "grid_ctas must be in [0, 65535] (got %d)", grid_ctas);
    if (!w || !seg_out) return fail(RMS_EINVAL, "w and seg_out must not be null");
    if (reinterpret_cast<uintptr_t>(w) % 16 || reinterpret_cast<uintptr_t>(seg_out) % 16)
        return fail(RMS_EALIGN, "w and seg_out must be 16-byte aligned");
    const int H = shape.H;
    const rms_shape local = {sp.row_end - sp.row_begin, 1, H};
    const int64_t R = local.T;
    const bool res = dh.ptr != nullptr;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t wb = (size_t)H * (w_dtype == RMS_FP32 ? 4 : 2);
    const size_t seg_bytes = (size_t)sp.n_seg * H * 8;
    if (R == 0) {  // a rank whose segments are all empty contributes zeros
        Span ins[1] = {span_of(w, wb, "w")};
        Span outs[1] = {span_of(seg_out, seg_bytes, "seg_out")};
        if ((rc = check_aliases(ins, 1, outs, 1))) return rc;
        cudaError_t e = cudaMemsetAsync(seg_out, 0, seg_bytes, st);
        return e == cudaSuccess ? ok() : cuda_fail(e, "cudaMemsetAsync(seg_out)");
    }
    if (!rstd) return fail(RMS_EINVAL, "rstd is null");
    if (reinterpret_cast<uintptr_t>(rstd) % 4) return fail(RMS_EALIGN, "rstd must be 4-byte aligned");
    Span ins[5], outs[2];
    int nin = 0;
    if ((rc = check_rows(local, x, res ? "h" : "x", false, &ins[nin++]))) return rc;
    if ((rc = check_rows(local, dy, "dy", false, &ins[nin++]))) return rc;
    if (res && (rc = check_rows(local, dh, "dh", false, &ins[nin++]))) return rc;
    ins[nin++] = span_of(w, wb, "w");
    ins[nin++] = span_of(rstd, (size_t)R * 4, "rstd");
    if ((rc = check_rows(local, dx, res ? "grad_h" : "dx", true, &outs[0]))) return rc;
    outs[1] = span_of(seg_out, seg_bytes, "seg_out");
    if ((rc = check_aliases(ins, nin, outs, 2))) return rc;
    if ((rc = check_workspace(ws, ws_size, sp.ws_bytes, ins, nin, outs, 2))) return rc;

    const Plan plan = det_plan(shape.T, H);  // the order of all rows
    rmsk::BwdParams p = {};
    p.R = (int32_t)R;
    p.heads = 1;
    p.H = H;
    p.nvec = H / 8;
    p.x = in_of(local, x);
    p.dy = in_of(local, dy);
    if (res) p.dh = in_of(local, dh);
    p.dx = out_of(local, dx);
    p.w = w;
    p.rstd = rstd;
    p.dw = nullptr;
    unsigned char* base = static_cast<unsigned char*>(ws);
    p.status = reinterpret_cast<unsigned*>(base);
    p.ticket = reinterpret_cast<unsigned*>(base + 4);
    p.acc = reinterpret_cast<double*>(base + kWsHeader);
    p.part = reinterpret_cast<double*>(base + kWsHeader + kAccBytes);
    p.block_rows = plan.B;
    p.blocks_per_chunk = plan.L;
    p.fold_segments = plan.S;
    p.n_chunks = sp.n_chunks;
    p.seg_len = plan.seg_len;
    p.seg_out = seg_out;
    p.n_seg_out = sp.n_seg;
    p.wait_cycles = g_wait_cycles.load();
    cudaError_t e = rmsk::launch_bwd_det(p, res, w_dtype == RMS_FP32, grid_ctas, st);
    if (e != cudaSuccess) return cuda_fail(e, "sharded backward launch");
    return ok();
}

}  // namespace

namespace rmsk {

int set_error(int code, const char* msg) {
    g_err = msg;
    return code;
}

int bwd_entry(rms_shape shape, rms_rows x, const void* w, int w_dtype, const float* rstd,
              rms_rows dy, const rms_rows* dh, rms_rows dx, float* dw, int deterministic,
              void* ws, size_t ws_bytes, int grid_ctas, void* stream, PreLaunchFn hook,
              void* hook_ctx) {
    return bwd_common(shape, x, w, w_dtype, rstd, dy, dh, dx, dw, deterministic, ws, ws_bytes,
                      grid_ctas, stream, 0, hook, hook_ctx);
}

int current_device() {
    int dev = 0;
    return cudaGetDevice(&dev) == cudaSuccess ? dev : -1;
}

int device_sm_count() {
    static PerDevice<1> cached;
    const int dev = current_device();
    if (dev < 0) return 148;
    return cached.get(dev, 0, [dev]() {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        return n;
    });
}

}  // namespace rmsk

extern "C" {

int rms_train_fwd(rms_shape shape, rms_rows x, const void* w, int w_dtype, rms_rows y,
                  float* rstd, float eps, void* stream) {
    int rc = check_shape(shape);
    if (rc) return rc;
    if (w_dtype != RMS_BF16 && w_dtype != RMS_FP32)
        return fail(RMS_EDTYPE, "w_dtype must be RMS_BF16 or RMS_FP32 (got %d)", w_dtype);
    const int64_t R = shape.T * shape.heads;
    if (R == 0) return ok();
    if (!w || !rstd) return fail(RMS_EINVAL, "w and rstd must not be null");
    if (reinterpret_cast<uintptr_t>(w) % 16) return fail(RMS_EALIGN, "w must be 16-byte aligned");
    if (reinterpret_cast<uintptr_t>(rstd) % 4) return fail(RMS_EALIGN, "rstd must be 4-byte aligned");
    Span ins[2], outs[2];
    if ((rc = check_rows(shape, x, "x", false, &ins[0]))) return rc;
    ins[1] = span_of(w, (size_t)shape.H * (w_dtype == RMS_FP32 ? 4 : 2), "w");
    if ((rc = check_rows(shape, y, "y", true, &outs[0]))) return rc;
    outs[1] = span_of(rstd, (size_t)R * 4, "rstd");
    if ((rc = check_aliases(ins, 2, outs, 2))) return rc;
    rmsk::FwdParams p = {};
    p.R = (int32_t)R;
    p.heads = shape.heads;
    p.H = shape.H;
    p.nvec = shape.H / 8;
    p.x = in_of(shape, x);
    p.y = out_of(shape, y);
    p.w = w;
    p.rstd = rstd;
    p.eps = eps;
    p.prefetch = fwd_prefetch(R, shape.H);
    cudaError_t e = rmsk::launch_fwd(p, false, w_dtype == RMS_FP32, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "forward launch");
}

int rms_residual_train_fwd(rms_shape shape, rms_rows x, rms_rows residual, const void* w,
                           int w_dtype, rms_rows h_out, rms_rows y, float* rstd, float eps,
                           void* stream) {
    int rc = check_shape(shape);
    if (rc) return rc;
    if (w_dtype != RMS_BF16 && w_dtype != RMS_FP32)
        return fail(RMS_EDTYPE, "w_dtype must be RMS_BF16 or RMS_FP32 (got %d)", w_dtype);
    const int64_t R = shape.T * shape.heads;
    if (R == 0) return ok();
    if (!w || !rstd) return fail(RMS_EINVAL, "w and rstd must not be null");
    if (reinterpret_cast<uintptr_t>(w) % 16) return fail(RMS_EALIGN, "w must be 16-byte aligned");
    if (reinterpret_cast<uintptr_t>(rstd) % 4) return fail(RMS_EALIGN, "rstd must be 4-byte aligned");
    Span ins[3], outs[3];
    if ((rc = check_rows(shape, x, "x", false, &ins[0]))) return rc;
    if ((rc = check_rows(shape, residual, "residual", false, &ins[1]))) return rc;
    ins[2] = span_of(w, (size_t)shape.H * (w_dtype == RMS_FP32 ? 4 : 2), "w");
    if ((rc = check_rows(shape, h_out, "h_out", true, &outs[0]))) return rc;
    if ((rc = check_rows(shape, y, "y", true, &outs[1]))) return rc;
    outs[2] = span_of(rstd, (size_t)R * 4, "rstd");
    if ((rc = check_aliases(ins, 3, outs, 3))) return rc;
    rmsk::FwdParams p = {};
    p.R = (int32_t)R;
    p.heads = shape.heads;
    p.H = shape.H;
    p.nvec = shape.H / 8;
    p.x = in_of(shape, x);
    p.res = in_of(shape, residual);
    p.h = out_of(shape, h_out);
    p.y = out_of(shape, y);
    p.w = w;
    p.rstd = rstd;
    p.eps = eps;
    p.prefetch = fwd_prefetch(R, shape.H);
    cudaError_t e = rmsk::launch_fwd(p, true, w_dtype == RMS_FP32, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? ok() : cuda_fail(e, "residual forward launch");
}

int rms_train_bwd(rms_shape shape, rms_rows x, const void* w, int w_dtype, const float* rstd,
                  rms_rows dy, rms_rows dx, float* dw, int deterministic, void* workspace,
                  size_t workspace_bytes, int grid_ctas, void* stream) {
    return bwd_common(shape, x, w, w_dtype, rstd, dy, nullptr, dx, dw, deterministic, workspace,
                      workspace_bytes, grid_ctas, stream);
}

int rms_residual_train_bwd(rms_shape shape, rms_rows h, const void* w, int w_dtype,
                           const float* rstd, rms_rows dy, rms_rows dh, rms_rows grad_h,
                           float* dw, int deterministic, void* workspace,
                           size_t workspace_bytes, int grid_ctas, void* stream) {
    return bwd_common(shape, h, w, w_dtype, rstd, dy, &dh, grad_h, dw, deterministic, workspace,
                      workspace_bytes, grid_ctas, stream);
}

int rms_train_bwd_accumulate(rms_shape shape, rms_rows x, const void* w, int w_dtype,
                             const float* rstd, rms_rows dy, rms_rows dx, float* dw,
                             int deterministic, void* workspace, size_t workspace_bytes,
                             int grid_ctas, void* stream) {
    return bwd_common(shape, x, w, w_dtype, rstd, dy, nullptr, dx, dw, deterministic, workspace,
                      workspace_bytes, grid_ctas, stream, 1);
}

int rms_residual_train_bwd_accumulate(rms_shape shape, rms_rows h, const void* w, int w_dtype,
                                      const float* rstd, rms_rows dy, rms_rows dh,
                                      rms_rows grad_h, float* dw, int deterministic,
                                      void* workspace, size_t workspace_bytes, int grid_ctas,
                                      void* stream) {
    return bwd_common(shape, h, w, w_dtype, rstd, dy, &dh, grad_h, dw, deterministic, workspace,
                      workspace_bytes, grid_ctas, stream, 1);
}

int rms_det_shard_plan(rms_shape shape, int rank, int world, int64_t* row_begin,
                       int64_t* row_end, size_t* workspace_bytes) {
    ShardPlan sp;
    const int rc = shard_plan(shape, rank, world, &sp);
    if (rc) return rc;
    if (row_begin) *row_begin = sp.row_begin;
    if (row_end) *row_end = sp.row_end;
    if (workspace_bytes) *workspace_bytes = sp.ws_bytes;
    return ok();
}

int rms_train_bwd_det_shard(rms_shape shape, int rank, int world, rms_rows x, const void* w,
                            int w_dtype, const float* rstd, rms_rows dy, rms_rows dh,
                            rms_rows dx, double* seg_out, void* workspace,
                            size_t workspace_bytes, int grid_ctas, void* stream) {
    return shard_common(shape, rank, world, x, w, w_dtype, rstd, dy, dh, dx, seg_out, workspace,
                        workspace_bytes, grid_ctas, stream);
}

int rms_det_fold_segments(rms_shape shape, const double* seg, float* dw, int accumulate,
                          void* stream) {
    int rc = check_shape(shape);
    if (rc) return rc;
    if (!seg || !dw) return fail(RMS_EINVAL, "seg and dw must not be null");
    if (reinterpret_cast<uintptr_t>(seg) % 16 || reinterpret_cast<uintptr_t>(dw) % 16)
        return fail(RMS_EALIGN, "seg and dw must be 16-byte aligned");
    const int H = shape.H;
    const int64_t R = shape.T * shape.heads;
    Span ins[1] = {span_of(seg, (size_t)kFoldSegments * H * 8, "seg")};
    Span outs[1] = {span_of(dw, (size_t)H * 4, "dw")};
    if ((rc = check_aliases(ins, 1, outs, 1))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (R == 0) {
        if (accumulate) return ok();
        cudaError_t e = cudaMemsetAsync(dw, 0, (size_t)H * 4, st);
        return e == cudaSuccess ? ok() : cuda_fail(e, "cudaMemsetAsync(dw)");
    }
    const Plan pl = det_plan(R, H);
    const int nonempty = (pl.n_chunks + pl.seg_len - 1) / pl.seg_len;
    cudaError_t e = rmsk::launch_fold_segments(seg, nonempty, H, dw, accumulate, st);
    return e == cudaSuccess ? ok() : cuda_fail(e, "fold launch");
}

size_t rms_train_bwd_workspace_bytes(rms_shape shape, int deterministic, int grid_ctas) {
    (void)grid_ctas;  // the layout does not depend on the grid
    if (check_shape(shape)) return 0;
    return ws_bytes(shape, deterministic);
}

int rms_det_plan(rms_shape shape, int32_t* block_rows, int32_t* blocks_per_chunk,
                 int32_t* fold_segments) {
    int rc = check_shape(shape);
    if (rc) return rc;
    const Plan p = det_plan(shape.T * shape.heads, shape.H);
    if (block_rows) *block_rows = p.B;
    if (blocks_per_chunk) *blocks_per_chunk = p.L;
    if (fold_segments) *fold_segments = p.S;
    return ok();
}

int rms_train_bwd_path(rms_shape shape, int deterministic) {
    int rc = check_shape(shape);
    if (rc) return rc;
    const int64_t R = shape.T * shape.heads;
    if (use_small(R, shape.H)) return 1;
    return deterministic ? 2 : 3;
}

int64_t rms_set_small_rows_limit(int64_t rows) {
    return g_small_rows_override.exchange(rows < 0 ? -1 : rows);
}

int rms_set_l2_prefetch(int rows) {
    return g_prefetch.exchange(rows < 0 ? -1 : rows);
}

int64_t rms_set_wait_limit_cycles(int64_t cycles) {
    return g_wait_cycles.exchange(cycles < 0 ? rmsk::kDefaultWaitCycles : cycles);
}

int rms_status(void* workspace, void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned word = 0;
    cudaError_t e;
    if (!workspace) {
        // the forward kernels take no workspace and have no device-side waits: only the
        // stream's own errors can be reported
        e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    } else {
        e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
        e = cudaMemcpy(&word, workspace, sizeof word, cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(status)");
        if (word) {
            e = cudaMemset(workspace, 0, sizeof word);
            if (e != cudaSuccess) return cuda_fail(e, "cudaMemset(status)");
        }
    }
    if (word) {
        if (word & rmsk::kStatusTimeout)
            return fail(RMS_ETIMEOUT, "a device-side bounded wait gave up (status 0x%x)", word);
        return fail(RMS_ECUDA, "device status 0x%x", word);
    }
    return ok();
}

const char* rms_last_error(void) { return g_err.c_str(); }

int rms_device_sms(void) { return rmsk::device_sm_count(); }

}  // extern "C"
