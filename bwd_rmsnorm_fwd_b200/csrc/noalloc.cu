// rms_train_bwd_noalloc: the blocked-FP32 (deterministic=0) backward with its scratch in
// a fixed device array owned by this library, for callers that cannot allocate device
// memory; rms_noalloc_status reads the device status word kept in that array.
//
// Who needs it: code that runs where cudaMalloc is not allowed or not available --
// inside a custom allocator's own callbacks, in a runtime that hands out only
// pre-planned buffers and forbids any further device allocation, or in a plugin whose
// host framework owns all device memory and gives it no way to ask for a workspace.
// Such a caller can still pass its inputs and outputs; this entry point needs nothing
// else.
//
// The scratch is one file-scope __device__ array of kScratchBytes (a 256-byte header
// holding the device status word and the CTA ticket, then FP64 accumulators for up to
// kMaxCols columns).  Every GPU that loads the library keeps this array until the
// process exits.  Host code cannot use the array's name as a device address, so the
// first call on each device (and the first after that device's context was replaced,
// e.g. by cudaDeviceReset) looks the address up with cudaGetSymbolAddress, with that
// device current, and caches it under the context's unique id; make that first call
// before any stream capture.  A call clears the ticket and the accumulators it uses, on
// the caller's stream, only once every host-side check has passed.  The status word is
// not cleared by calls: once a bounded wait has given up it stays set until
// rms_noalloc_status reads it.  All calls share the one array: two calls whose work
// overlaps on the GPU (different streams, or different host threads without ordering)
// race on it and produce wrong dw.
#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "rmsnorm_train.h"

namespace {

constexpr int kMaxCols = 8192;
constexpr size_t kHeaderBytes = 256;   // status word at 0, CTA ticket at 4
constexpr size_t kTicketOffset = 4;
constexpr size_t kScratchBytes = kHeaderBytes + (size_t)kMaxCols * sizeof(double);  // 65,792

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// ---- the context of the calling thread, through the driver's entry points ---------------
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

template <typename F>
F driver_fn(const char* name) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<F>(p);
}

// Unique id of the current context (0 when none is current or the query is unavailable).
unsigned long long current_context_id() {
    static CtxGetCurrentFn get_cur = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
    if (!get_cur || !get_id) return 0;
    CUcontext c = nullptr;
    unsigned long long id = 0;
    if (get_cur(&c) != CUDA_SUCCESS || !c || get_id(c, &id) != CUDA_SUCCESS) return 0;
    return id;
}

using rmsk::kMaxDevices;
struct DeviceScratch {
    unsigned long long ctx_id;  // context the address belongs to
    void* addr;
};
DeviceScratch g_dev[kMaxDevices];
std::mutex g_setup_mutex;

// Device address of g_scratch in the current device's context, looked up once per device
// and context.
int scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return rmsk::set_error(RMS_ECUDA, "rms_train_bwd_noalloc: cudaGetDevice failed");
    if (dev < 0 || dev >= kMaxDevices)
        return rmsk::set_error(RMS_EINVAL, "rms_train_bwd_noalloc: device index beyond 63");
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    const unsigned long long id = current_context_id();
    DeviceScratch& d = g_dev[dev];
    if (!d.addr || id == 0 || d.ctx_id != id) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
        if (e != cudaSuccess || !p) {
            char msg[200];
            snprintf(msg, sizeof msg, "rms_train_bwd_noalloc: cudaGetSymbolAddress failed: %s",
                     cudaGetErrorString(e));
            return rmsk::set_error(RMS_ECUDA, msg);
        }
        d.addr = p;
        d.ctx_id = current_context_id();  // the lookup makes the primary context current
    }
    *out = d.addr;
    return RMS_OK;
}

struct ClearScratch {
    unsigned char* scratch;
    size_t bytes;  // ticket up to the last accumulator of the call
};

// The ticket and the call's accumulators must start at zero (the status word is left as is).
int clear_scratch(void* ctx, cudaStream_t s) {
    const ClearScratch* c = static_cast<const ClearScratch*>(ctx);
    if (cudaMemsetAsync(c->scratch + kTicketOffset, 0, c->bytes, s) != cudaSuccess)
        return rmsk::set_error(RMS_ECUDA, "rms_train_bwd_noalloc: clearing the scratch failed");
    return RMS_OK;
}

}  // namespace

extern "C" int rms_train_bwd_noalloc(rms_shape shape, rms_rows x, const void* w, int w_dtype,
                                     const float* rstd, rms_rows dy, rms_rows dx, float* dw,
                                     void* stream) {
    if (shape.H > kMaxCols) {
        char msg[160];
        snprintf(msg, sizeof msg,
                 "rms_train_bwd_noalloc: H = %d exceeds the fixed scratch of %d columns",
                 shape.H, kMaxCols);
        return rmsk::set_error(RMS_EINVAL, msg);
    }
    const size_t need = rms_train_bwd_workspace_bytes(shape, 0, 0);
    if (need == 0)  // invalid shape: the regular entry point reports why
        return rms_train_bwd(shape, x, w, w_dtype, rstd, dy, dx, dw, 0, nullptr, 0, 0, stream);
    if (need > kScratchBytes)
        return rmsk::set_error(RMS_EINVAL, "rms_train_bwd_noalloc: shape needs more scratch "
                                           "than the fixed array holds");
    void* scratch = nullptr;
    int rc = scratch_address(&scratch);
    if (rc != RMS_OK) return rc;
    ClearScratch c = {static_cast<unsigned char*>(scratch),
                      kHeaderBytes - kTicketOffset + (size_t)shape.H * sizeof(double)};
    return rmsk::bwd_entry(shape, x, w, w_dtype, rstd, dy, nullptr, dx, dw, 0, scratch,
                           kScratchBytes, 0, stream, clear_scratch, &c);
}

extern "C" int rms_noalloc_status(void* stream) {
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) {
        char msg[200];
        snprintf(msg, sizeof msg, "cudaStreamSynchronize: %s", cudaGetErrorString(e));
        return rmsk::set_error(RMS_ECUDA, msg);
    }
    void* scratch = nullptr;
    int rc = scratch_address(&scratch);
    if (rc != RMS_OK) return rc;
    unsigned word = 0;
    e = cudaMemcpy(&word, scratch, sizeof word, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return rmsk::set_error(RMS_ECUDA, "reading the status word failed");
    if (!word) return rmsk::set_error(RMS_OK, "");
    e = cudaMemset(scratch, 0, sizeof word);
    if (e != cudaSuccess) return rmsk::set_error(RMS_ECUDA, "clearing the status word failed");
    char msg[160];
    if (word & rmsk::kStatusTimeout) {
        snprintf(msg, sizeof msg,
                 "a device-side bounded wait of rms_train_bwd_noalloc gave up (status 0x%x)",
                 word);
        return rmsk::set_error(RMS_ETIMEOUT, msg);
    }
    snprintf(msg, sizeof msg, "device status 0x%x", word);
    return rmsk::set_error(RMS_ECUDA, msg);
}
