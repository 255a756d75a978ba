/*
 * librmsnorm_train -- training RMSNorm for NVIDIA B200 (sm_100a), C ABI.
 *
 * The operation (flashinfer PR #8848 "...sm_100a non-deterministic backward...",
 * introduction and "Measurement"/"Workload"; flashinfer PR #8512 "fix(cake_rmsnorm_det):
 * fixed-order dw for the smallest token counts of the SM100/SM103 backward", introduction):
 *
 *   forward   rstd_r = 1 / sqrt(mean_j(x_rj^2) + eps)          FP32 [R]
 *             y_rj   = x_rj * rstd_r * w_j                      BF16, x's layout
 *   backward  xh = x * rstd, g = dy * w, c_r = (1/H) sum_j g_rj xh_rj
 *             dx_rj  = rstd_r * (g_rj - xh_rj * c_r)            BF16
 *             dw_j   = sum_r dy_rj * xh_rj                      FP32 [H]
 *   residual  h = BF16(x + residual) and the forward runs on h (h is returned);
 *             the backward takes dy and dh and returns grad_h = BF16(dh + dx)
 *             (PR #8512 introduction, "Residual rows"; PR #8848 "Key").
 *
 * Two backward modes (PR #8512 introduction; PR #8848 introduction):
 *   deterministic != 0  every dw column is summed over a fixed row order with exact
 *                       products and TwoSum compensation, the pieces are folded in a
 *                       fixed FP64 order and rounded once to FP32.  The order depends
 *                       only on (rows, H) -- never on grid_ctas or the SM count -- so dw
 *                       is bit-identical across grids; rms_det_plan() returns it.
 *   deterministic == 0  blocked FP32 sums (eight rows per block) per thread, combined
 *                       in FP64 across the grid in arrival order.
 *
 * Layout.  A row tensor is a [T, heads, H] view: row (t, k) starts at element
 * ptr + t*st + k*sk and its H elements are contiguous.  Rows are numbered
 * r = t*heads + k (R = T*heads); rstd is a dense FP32 [R] array in that order.
 * Per-head views such as [T,24,256] with strides (12288, 512, 1) or dense
 * [T,4,256] share one w[H] (PR #8848 introduction; PR #8512 squashed commit of #8626).
 * x/y/dy/dx/h/residual/dh/grad_h are BF16; w is BF16 or FP32; dw is FP32.
 *
 * Requirements (checked on the host before anything is launched; a failing call
 * writes nothing):  1 <= H <= 8192, H % 8 == 0; heads >= 1; T >= 0; T*heads < 2^31;
 * every row pointer, w and dw 16-byte aligned; st and sk multiples of 8 elements;
 * rstd 4-byte aligned; no output range overlaps an input range or another output
 * (dw aliasing w is rejected, PR #8512 review "Reject dw that aliases w").
 *
 * Ownership.  The caller owns every buffer, the workspace included.  The library
 * allocates no device memory, never synchronises inside the compute calls, and
 * launches only 1-D grids (PR #8848 review "Reject non-one-dimensional grids").
 * All calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default).
 *
 * Errors.  Every entry point returns RMS_OK or a negative code; rms_last_error()
 * gives a message (thread-local).  Launch failures return RMS_ECUDA.  Conditions the
 * device detects are written to the workspace status word; rms_status() reads them.
 */
#ifndef RMSNORM_TRAIN_H
#define RMSNORM_TRAIN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element types: BF16 (bfloat16 bits) or FP32. */
enum { RMS_BF16 = 0, RMS_FP32 = 1 };

/* Return codes. */
enum {
    RMS_OK = 0,
    RMS_EINVAL = -1,     /* bad shape, null pointer, bad stride, bad grid_ctas   */
    RMS_EDTYPE = -2,     /* unsupported dtype code                                 */
    RMS_EALIGN = -3,     /* pointer or stride not aligned as required               */
    RMS_EALIAS = -4,     /* an output overlaps an input or another output           */
    RMS_EWORKSPACE = -5, /* workspace missing or smaller than the size query says   */
    RMS_ECUDA = -6,      /* a CUDA runtime call or launch failed                    */
    RMS_ETIMEOUT = -7    /* a device-side bounded wait gave up (rms_status)         */
};

/* A [T, heads, H] row view; strides in elements, innermost stride 1. */
typedef struct {
    void* ptr;
    int64_t st; /* stride between tokens t   */
    int64_t sk; /* stride between heads k    */
} rms_rows;

typedef struct {
    int64_t T;     /* tokens (rows per head) */
    int32_t heads; /* rows per token         */
    int32_t H;     /* row width              */
} rms_shape;

/* Forward.  Reads x [T,heads,H] BF16 and w [H] (w_dtype), writes y (BF16, its own
 * strides) and rstd (FP32 [R]).  eps is added to the mean of squares (1e-6 on the
 * pages, PR #8848 "Workload").  T == 0 is a no-op. */
int rms_train_fwd(rms_shape shape, rms_rows x, const void* w, int w_dtype, rms_rows y,
                  float* rstd, float eps, void* stream);

/* Residual forward.  h_out = BF16(x + residual); then the forward of rms_train_fwd on
 * h_out.  Writes h_out, y and rstd. */
int rms_residual_train_fwd(rms_shape shape, rms_rows x, rms_rows residual, const void* w,
                           int w_dtype, rms_rows h_out, rms_rows y, float* rstd, float eps,
                           void* stream);

/* Backward.  Reads x (the forward's input), w, rstd (the forward's FP32 output) and dy;
 * writes dx (BF16) and dw (FP32 [H], overwritten, not accumulated).  The formulas are
 * the gradient of the forward (PR #8848 introduction: dx BF16, dw FP32); the two dw
 * modes are those of the file preamble (deterministic: PR #8512 introduction;
 * deterministic == 0: PR #8848 introduction and its review on blocked FP32 sums).
 * The workspace (>= rms_train_bwd_workspace_bytes(shape, deterministic, grid_ctas)
 * bytes, 256-byte aligned) must be zero-filled once before its first use; every call
 * leaves it ready for the next.  Calls sharing a workspace must be stream-ordered.
 * grid_ctas = 0 picks the grid; any other value (1 .. 65535) sets the CTA count of the
 * main backward kernel and never changes the deterministic dw bits (PR #8512
 * introduction: dw independent of the grid and the SM count).  T == 0 writes dw = 0. */
int rms_train_bwd(rms_shape shape, rms_rows x, const void* w, int w_dtype, const float* rstd,
                  rms_rows dy, rms_rows dx, float* dw, int deterministic, void* workspace,
                  size_t workspace_bytes, int grid_ctas, void* stream);

/* Residual backward (PR #8512 introduction, "Residual rows": the backward takes the
 * gradients of y and of h and returns the gradient of h; PR #8848 "Key").  h is the
 * forward's h_out; dy the gradient of y, dh the gradient of h.  Writes
 * grad_h = BF16(dh + dx), one rounding of the FP32 sum, and dw.  Workspace rules as
 * rms_train_bwd. */
int rms_residual_train_bwd(rms_shape shape, rms_rows h, const void* w, int w_dtype,
                           const float* rstd, rms_rows dy, rms_rows dh, rms_rows grad_h,
                           float* dw, int deterministic, void* workspace,
                           size_t workspace_bytes, int grid_ctas, void* stream);

/* Backward with gradient accumulation: rms_train_bwd / rms_residual_train_bwd, except that
 * dw is read as well as written: dw = FP32(dw + dw_call), where dw_call is exactly what the
 * overwrite call returns for the same inputs and mode (one FP32 addition of the call's
 * rounded FP32 sum).  So the deterministic mode's accumulated bits depend only on the
 * previous dw bits and the inputs.  Used to sum dw over the micro-batches of a step or the
 * row shards of a batch without a separate add kernel (the pages' checkpointed training
 * step, PR #8848 "Key", gives the setting; the pages return dw and do not accumulate).
 * T == 0 leaves dw unchanged.  Other arguments, checks and outputs as the overwrite calls. */
int rms_train_bwd_accumulate(rms_shape shape, rms_rows x, const void* w, int w_dtype,
                             const float* rstd, rms_rows dy, rms_rows dx, float* dw,
                             int deterministic, void* workspace, size_t workspace_bytes,
                             int grid_ctas, void* stream);
int rms_residual_train_bwd_accumulate(rms_shape shape, rms_rows h, const void* w, int w_dtype,
                                      const float* rstd, rms_rows dy, rms_rows dh,
                                      rms_rows grad_h, float* dw, int deterministic,
                                      void* workspace, size_t workspace_bytes, int grid_ctas,
                                      void* stream);

/* Backward without any device allocation: the deterministic == 0 backward of
 * rms_train_bwd, whose scratch (status word, CTA ticket and FP64 accumulators for up to
 * 8192 columns: 65,792 bytes) lives in one fixed device array inside this library
 * instead of a caller-allocated workspace.  The pages have no counterpart; it exists for
 * callers that cannot allocate device memory at all -- code running inside an
 * allocator's callbacks, runtimes that hand out only pre-planned buffers, plugins whose
 * host owns every device buffer -- and so cannot provide a workspace.  The caller still
 * passes every input and output.  H above 8192 is rejected with RMS_EINVAL.  The first
 * call on each device (and the first after its context was replaced, e.g. by
 * cudaDeviceReset) looks up the array's device address (cudaGetSymbolAddress with that
 * device current); make that first call before any stream capture.  A call that passes
 * every host-side check clears the ticket and the accumulators it uses on `stream`; a
 * rejected call queues nothing.  Every GPU that loaded the library keeps the array
 * until the process exits.  All calls share the one array, so calls whose work overlaps
 * on the GPU (other streams, unordered threads) race and corrupt dw.  A bounded device
 * wait that gives up (see rms_set_wait_limit_cycles) leaves the call's outputs invalid
 * and sets the array's status word, which stays set across later calls until
 * rms_noalloc_status reads it.  Other arguments, checks and outputs are those of
 * rms_train_bwd. */
int rms_train_bwd_noalloc(rms_shape shape, rms_rows x, const void* w, int w_dtype,
                          const float* rstd, rms_rows dy, rms_rows dx, float* dw, void* stream);

/* Status of rms_train_bwd_noalloc on the current device (no counterpart on the pages):
 * synchronises `stream`, then reads and clears the status word of the library's fixed
 * scratch array.  Returns RMS_OK, RMS_ETIMEOUT (a bounded wait of an earlier call gave up:
 * that call's dx and dw are invalid) or RMS_ECUDA. */
int rms_noalloc_status(void* stream);

/* Workspace bytes the backward needs for this shape, mode and grid (0 on bad input).
 * The workspace holds counters and accumulators only, never rows: a status word, the CTA
 * ticket, an FP64 accumulator kept zero between calls, and, for the deterministic pair,
 * the FP64 chunk partials (PR #8512 review summary, "Column-task workspace handling":
 * counters only, no partial-row capacity). */
size_t rms_train_bwd_workspace_bytes(rms_shape shape, int deterministic, int grid_ctas);

/* The fixed deterministic summation order for this shape: rows are cut into blocks of
 * *block_rows; each block is summed in row order with exact products and TwoSum and
 * converted to FP64 (sum + compensation); *blocks_per_chunk consecutive blocks are
 * folded left to right in FP64 into one chunk partial; the chunk partials are cut into
 * *fold_segments contiguous segments of ceil(chunks / segments) chunks, each folded left
 * to right, and the segment sums are folded left to right and rounded once to FP32.
 * Returns RMS_OK or RMS_EINVAL. */
int rms_det_plan(rms_shape shape, int32_t* block_rows, int32_t* blocks_per_chunk,
                 int32_t* fold_segments);

/* Row-sharded deterministic backward (PR #8512 introduction: the fixed row order, the
 * fixed-order FP64 fold and the single FP32 rounding, extended across GPUs; the pages run one
 * GPU).  The T rows of a [T, H] problem (heads == 1) are split over `world` ranks (world
 * divides 16): rank r owns fold segments [r*16/world, (r+1)*16/world) of the plan of all T
 * rows (rms_det_plan), which are whole chunks of contiguous rows [row_begin, row_end).
 * Folding every rank's segment sums in segment order gives dw bit-identical to the
 * single-GPU deterministic backward of all T rows.
 *
 * rms_det_shard_plan: the rows of `rank` and the workspace bytes its shard call needs. */
int rms_det_shard_plan(rms_shape shape, int rank, int world, int64_t* row_begin,
                       int64_t* row_end, size_t* workspace_bytes);

/* rms_train_bwd_det_shard: the deterministic backward of rank `rank`'s rows.  `shape` is the
 * whole problem's [T, 1, H]; x (or h), dy, dh, dx and rstd hold only the rank's
 * row_end - row_begin rows (views with st = their own row stride).  dh.ptr == NULL selects
 * the plain form, otherwise the residual form (dx is then grad_h).  Writes dx and, instead
 * of dw, the FP64 sums of the rank's 16/world segments to seg_out [16/world][H] (16-byte
 * aligned; 0 for an empty segment).  Workspace as rms_det_shard_plan says, zero-filled once,
 * as for rms_train_bwd.  The caller gathers every rank's seg_out in rank order into a
 * [16][H] table (an all-gather; NCCL over NVLink on GPUs) and calls rms_det_fold_segments. */
int rms_train_bwd_det_shard(rms_shape shape, int rank, int world, rms_rows x, const void* w,
                            int w_dtype, const float* rstd, rms_rows dy, rms_rows dh,
                            rms_rows dx, double* seg_out, void* workspace,
                            size_t workspace_bytes, int grid_ctas, void* stream);

/* rms_det_fold_segments: folds the [16][H] FP64 table of segment sums of the whole problem
 * `shape` left to right per column (its non-empty segments) and rounds once to FP32 into dw
 * (dw = FP32(dw + that value) when accumulate != 0).  T == 0 writes dw = 0 (or leaves it). */
int rms_det_fold_segments(rms_shape shape, const double* seg, float* dw, int accumulate,
                          void* stream);

/* Which backward program a call with this shape runs: 1 = single-launch small-row
 * kernel (row tasks + column tasks), 2 = main kernel + fixed-order fold kernel
 * (deterministic), 3 = single kernel with FP64 grid combine (non-deterministic).
 * Negative on bad input. */
int rms_train_bwd_path(rms_shape shape, int deterministic);

/* Largest row count R (= T*heads) served by the single-launch small-row program; the
 * default is chosen from H.  Setting a value >= 0 overrides it for every later call
 * in this process (not thread-safe against concurrent backward calls); -1 restores
 * the default.  Returns the previous override (-1 if none). */
int64_t rms_set_small_rows_limit(int64_t rows);

/* L2 prefetch of rows ahead of the forward's own loads (PR #8656 introduction: one bulk L2
 * prefetch per tensor of the CTA's next row block).  rows > 0: the forward's one-CTA-per-row
 * kernel (H > 1024) warms that many of the CTA's next rows (x, and the residual); 0 turns it
 * off; -1 restores the library's choice (one row ahead below 32768 rows, none above, as
 * measured).  Affects later calls in this process (not thread-safe against concurrent
 * calls); never changes results.  Returns the previous setting. */
int rms_set_l2_prefetch(int rows);

/* Limit, in SM clock cycles, of every device-side wait of later launches in this
 * process (the backward's bulk-copy pipeline barrier waits; the forward has none); the
 * default is about two seconds.  A wait that reaches it makes the kernel record
 * RMS_ETIMEOUT in its workspace status word (see rms_status) and finish without waiting
 * further; its outputs are then invalid.  Shorter limits exist to test that path (0
 * makes every wait a single non-blocking probe); a negative value restores the default.
 * Returns the previous limit.  Not thread-safe against concurrent launches. */
int64_t rms_set_wait_limit_cycles(int64_t cycles);

/* Synchronises `stream` and reads and clears the device status word of `workspace`
 * (written by the backward when a bounded device wait gives up; the pages have no
 * counterpart).  With workspace == NULL it only synchronises: the forward takes no
 * workspace and has no device-side waits, so the stream's own errors are all there is to
 * report.  Returns RMS_OK, RMS_ETIMEOUT or RMS_ECUDA. */
int rms_status(void* workspace, void* stream);

/* Message for the last non-zero return on this thread ("" if none). */
const char* rms_last_error(void);

/* Number of SMs of the current device (0 on error). */
int rms_device_sms(void);

#ifdef __cplusplus
}
#endif

#endif /* RMSNORM_TRAIN_H */
