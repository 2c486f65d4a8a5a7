// dsc_static_bwd_noalloc: the static-convolution backward without caller-provided
// workspace, for callers that cannot allocate device memory.
//
// dsc_static_bwd needs scratch for its per-block weight-gradient partials, which the
// caller normally allocates and passes in.  Some callers cannot: a plug-in handed only
// its input and output buffers by a host framework that owns every device allocation,
// or a latency-critical loop where cudaMalloc (which may synchronise the device) is
// not acceptable.  This entry point takes its scratch from a fixed array compiled into
// the library instead, and allocates nothing.
//
// The array lives in device global memory as a file-scope __device__ variable; every
// GPU that loads the library holds it until the process exits.  Host code cannot use
// the array's name as a device address (on the host it names a stand-in object), so
// each call looks the address up with cudaGetSymbolAddress, with the calling device
// current, and passes it to the kernels.  The lookup is a host-side query; doing it
// on every call (rather than caching it) keeps the address right after the device's
// context is torn down and the module is loaded again, for example after
// cudaDeviceReset.
#include <cstdio>

#include "../../include/dsc.h"
#include "internal.h"

namespace {

constexpr size_t kScratchBytes = 16u << 20;   // 16 MiB

__device__ __align__(256) float g_static_bwd_scratch[kScratchBytes / sizeof(float)];

// Address of the scratch array on the current device.  Returns nullptr (and records
// why) on failure.  The first call on a device may load the library's module onto it.
float *scratch_on_current_device() {
    float *ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress((void **)&ptr, g_static_bwd_scratch);
    if (e != cudaSuccess || !ptr) {
        char msg[256];
        snprintf(msg, sizeof(msg), "dsc_static_bwd_noalloc: cudaGetSymbolAddress failed: %s",
                 cudaGetErrorString(e));
        dsc::set_last_error(msg);
        return nullptr;
    }
    return ptr;
}

}  // namespace

extern "C" {

DSC_API size_t dsc_static_bwd_noalloc_max_scratch_bytes(void) { return kScratchBytes; }

DSC_API dsc_status_t dsc_static_bwd_noalloc(const void *x, const void *w, const void *dy,
                                            void *dx, float *dw, int B, int T, int D, int W,
                                            dsc_dtype_t dt, dsc_stream_t stream) {
    // Same argument rules as dsc_static_bwd (checked there too, with its own messages);
    // the needed scratch is the size dsc_static_bwd_workspace_bytes reports.
    const size_t need = dsc_static_bwd_workspace_bytes(B, T, D, W, dt);
    if (need == 0) {
        // Invalid sizes or dtype: let dsc_static_bwd classify and report them.
        return dsc_static_bwd(x, w, dy, dx, dw, nullptr, 0, B, T, D, W, dt, stream);
    }
    if (need > kScratchBytes) {
        char msg[256];
        snprintf(msg, sizeof(msg),
                 "dsc_static_bwd_noalloc: these sizes need %zu bytes of scratch, above the fixed "
                 "%zu-byte array; use dsc_static_bwd with a caller-provided workspace",
                 need, kScratchBytes);
        dsc::set_last_error(msg);
        return DSC_ERR_UNSUPPORTED;
    }
    float *scratch = scratch_on_current_device();
    if (!scratch) return DSC_ERR_CUDA;
    // Every partial slot the reduction reads is written earlier in the same call, so
    // nothing in the array has to start at zero.
    return dsc_static_bwd(x, w, dy, dx, dw, scratch, kScratchBytes, B, T, D, W, dt, stream);
}

}  // extern "C"
