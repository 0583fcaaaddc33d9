// ssm_selective_scan_fwd_noalloc: the selective-scan forward with scratch memory
// that the library owns, for callers that cannot allocate device memory.
//
// Who needs it: code that runs where a cudaMalloc is not allowed or not wanted,
// e.g. a host runtime that hands out only fixed, preallocated buffers, a caller
// without access to an allocator (a plain C program embedded in another runtime
// that owns device memory), or a latency-critical loop that must not risk the
// implicit device synchronisation a cudaMalloc can cause. Such callers still pass
// their inputs and outputs; only the scan's scratch (two-pass chunk summaries,
// the bidirectional fp32 partial) moves into a fixed array compiled into the
// library.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "../../include/ssm.h"
#include "launch.h"

namespace {

// The scratch array: one per GPU that loads the library, held until the process
// exits. In host code its name is only a stand-in; the device address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SSM_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 256;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per
// device (with that device current) and cached.
cudaError_t scratch_on_current_device(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" ssm_status_t ssm_selective_scan_fwd_noalloc(const ssm_scan_args_t* args,
                                                       ssm_stream_t stream) {
    size_t need = 0;
    ssm_status_t st = ssm_selective_scan_workspace_size(args, &need);
    if (st != SSM_OK) return st;
    if (need > (size_t)SSM_NOALLOC_SCRATCH_BYTES) {
        char msg[200];
        snprintf(msg, sizeof(msg),
                 "this call needs %zu bytes of scratch; the fixed no-allocation scratch holds "
                 "%zu bytes (use ssm_selective_scan_fwd with a caller workspace)",
                 need, (size_t)SSM_NOALLOC_SCRATCH_BYTES);
        ssm::set_error_detail(msg);
        return SSM_ERR_WORKSPACE;
    }
    ssm_scan_args_t a = *args;
    a.workspace = nullptr;
    a.workspace_bytes = 0;
    if (need > 0) {
        void* p = nullptr;
        cudaError_t e = scratch_on_current_device(&p);
        if (e != cudaSuccess) {
            char msg[200];
            snprintf(msg, sizeof(msg), "cudaGetSymbolAddress of the scratch array: %s",
                     cudaGetErrorString(e));
            ssm::set_error_detail(msg);
            return SSM_ERR_CUDA;
        }
        a.workspace = p;
        a.workspace_bytes = (size_t)SSM_NOALLOC_SCRATCH_BYTES;
    }
    return ssm_selective_scan_fwd(&a, stream);
}
