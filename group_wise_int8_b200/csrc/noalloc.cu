// wino_conv2d_int8_noalloc: the convolution of wino_conv2d_int8 for callers
// that cannot allocate device memory.
//
// Some callers have no way to obtain a device workspace: code running where
// cudaMalloc is forbidden or unavailable (inside a real-time or embedded loop
// that must not touch the allocator, a plugin whose host framework owns all
// device memory, or a caller that cannot carry an extra buffer through its
// interface).  For them the workspace lives in a fixed array in the library's
// own device memory, sized kNoAllocScratchBytes; every GPU that loads the
// library keeps that array for the life of the process.
//
// The host cannot use the array's name as a device address (in host code it
// names a host-side stand-in), so the device address is looked up once per
// device with cudaGetSymbolAddress, with that device current, on the first
// call made on it.  That first call therefore does a runtime lookup, and it
// should happen before any stream capture begins.
//
// All calls share the one array and it keeps whatever the previous call left
// there.  The convolution itself clears everything that must start at zero
// (the Y absmax table and the device error word) at the start of each call, so
// leftover contents never change a result.  The error word of the last call
// lives in the array too: wino_check_device_error_noalloc reads it (after that
// call and before the next one, which clears it).  Two calls whose kernels overlap
// on the GPU (different streams, or different host threads without ordering)
// race on the array and corrupt each other's intermediates: serialise them.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/wino.h"

namespace {

constexpr size_t kNoAllocScratchBytes = WINO_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// The scratch array: workspace of every wino_conv2d_int8_noalloc call.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once per device).
int scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return WINO_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return WINO_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return WINO_OK;
}

}  // namespace

extern "C" int wino_conv2d_int8_noalloc(wino_plan_t plan, const void* x_dev, int x_dtype, int N, int H, int W,
                                        int Cin, const void* wt_dev, int Cout, void* y_dev, int y_dtype,
                                        void* stream) {
    if (!plan) return WINO_ERR_INVALID_ARG;
    const size_t need = wino_workspace_bytes(plan, N, H, W, Cin, Cout);
    if (need == 0) return WINO_ERR_INVALID_ARG;
    if (need > kNoAllocScratchBytes) return WINO_ERR_WORKSPACE;
    void* scratch = nullptr;
    const int rc = scratch_address(&scratch);
    if (rc != WINO_OK) return rc;
    return wino_conv2d_int8(plan, x_dev, x_dtype, N, H, W, Cin, wt_dev, Cout, y_dev, y_dtype, scratch,
                            kNoAllocScratchBytes, stream);
}

extern "C" int wino_check_device_error_noalloc(wino_plan_t plan, int N, int H, int W, int Cin, int Cout,
                                               void* stream) {
    if (!plan) return WINO_ERR_INVALID_ARG;
    const size_t need = wino_workspace_bytes(plan, N, H, W, Cin, Cout);
    if (need == 0) return WINO_ERR_INVALID_ARG;
    if (need > kNoAllocScratchBytes) return WINO_ERR_WORKSPACE;
    void* scratch = nullptr;
    const int rc = scratch_address(&scratch);
    if (rc != WINO_OK) return rc;
    return wino_check_device_error(plan, scratch, N, H, W, Cin, Cout, stream);
}
