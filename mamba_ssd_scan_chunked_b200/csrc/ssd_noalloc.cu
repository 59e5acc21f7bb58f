// Prefill entry point for callers that cannot allocate device memory.
//
// ssd_chunk_scan_fwd needs a caller-provided workspace (the per-token dt and
// decay cumsum, the fp32 states handed from chunk to chunk, progress flags).
// Some callers cannot obtain one: code that may only use the input and output
// buffers it was handed, for instance a plugin inside a host framework that
// owns all device memory, or a latency-critical path where cudaMalloc (which
// can synchronise the device) is not allowed.  This entry point instead uses a
// fixed scratch array that lives in the library's own device memory.  It is
// reserved on a device when the library's device code is loaded there (with
// lazy module loading: at the first address lookup below) and stays until the
// process exits.
#include <mutex>

#include "../../include/ssd.h"
#include "ssd_internal.h"

namespace ssd {

// The scratch.  In host code `g_noalloc_scratch` is only a host-side stand-in
// for the symbol, not a device address: the device address is obtained with
// cudaGetSymbolAddress below, once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SSD_NOALLOC_WORKSPACE_BYTES];

static std::mutex g_noalloc_mutex;
static void* g_noalloc_ptr[64];

// Device address of the scratch on the current device (looked up on the first
// call made with that device current, then cached for the life of the process:
// a device reset would leave the cached address stale).
static cudaError_t noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return cudaSuccess;
}

}  // namespace ssd

extern "C" ssd_status_t ssd_chunk_scan_fwd_noalloc(const ssd_prefill_desc_t* desc, const void* x, const void* dt_raw,
                                                   const float* dt_bias, const float* A, const void* B, const void* C,
                                                   const float* D, const void* init_state, void* y, void* final_state,
                                                   void* stream) {
    size_t need = 0;
    const ssd_status_t st = ssd_chunk_scan_workspace_size(desc, &need);
    if (st != SSD_OK) return st;
    if (need > SSD_NOALLOC_WORKSPACE_BYTES) return SSD_ERR_WORKSPACE;   // problem too large for the scratch
    void* scratch = nullptr;
    if (ssd::noalloc_scratch(&scratch) != cudaSuccess) return SSD_ERR_CUDA;
    return ssd_chunk_scan_fwd(desc, x, dt_raw, dt_bias, A, B, C, D, init_state, y, final_state, scratch,
                              SSD_NOALLOC_WORKSPACE_BYTES, stream);
}
