// rms_train_bwd_noalloc: the blocked-FP32 (deterministic=0) backward with its scratch in
// a fixed device array owned by this library, for callers that cannot allocate device
// memory.
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
// first call on each device looks the address up with cudaGetSymbolAddress (with that
// device current) and caches it; make that first call before any stream capture.
// Every call clears the part of the array that must start at zero, on the caller's
// stream.  All calls share the one array: two calls whose work overlaps on the GPU
// (different streams, or different host threads without ordering) race on it and
// produce wrong dw.
#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "rmsnorm_train.h"

namespace {

constexpr int kMaxCols = 8192;
constexpr size_t kHeaderBytes = 256;
constexpr size_t kScratchBytes = kHeaderBytes + (size_t)kMaxCols * sizeof(double);  // 65,792

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices];
std::mutex g_setup_mutex;

// Device address of g_scratch on the current device, looked up once per device.
int scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return RMS_ECUDA;
    if (dev < 0 || dev >= kMaxDevices) return RMS_EINVAL;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_scratch);
        if (e != cudaSuccess || !p) return RMS_ECUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
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
    if (scratch_address(&scratch) != RMS_OK)
        return rmsk::set_error(RMS_ECUDA, "rms_train_bwd_noalloc: cudaGetSymbolAddress failed");
    // the status word, the ticket and the accumulators must start at zero
    cudaError_t e = cudaMemsetAsync(scratch, 0, need, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return rmsk::set_error(RMS_ECUDA, "rms_train_bwd_noalloc: clearing the scratch failed");
    return rms_train_bwd(shape, x, w, w_dtype, rstd, dy, dx, dw, 0, scratch, kScratchBytes, 0,
                         stream);
}
