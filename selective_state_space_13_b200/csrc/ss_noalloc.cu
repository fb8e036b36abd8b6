// selective_scan_fwd_noalloc: the selective scan for callers that cannot allocate device memory.
//
// The scratch that segmented scans (segment carries) and multi-direction scans (fp32
// per-direction outputs) need lives in one fixed array of this library's device memory instead
// of a caller-provided workspace.  The array is a file-scope __device__ variable, so every GPU
// that loads the library holds SS_NOALLOC_SCRATCH_BYTES of it until the process exits.
//
// Host code never passes the array's name to a kernel: in host code that name is only a
// stand-in for the device symbol.  Its device address is looked up once per device with
// cudaGetSymbolAddress (with that device current) on the first call made on that device.
#include <cuda_runtime.h>

#include <mutex>

#include "ss_internal.h"

namespace {

constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[SS_NOALLOC_SCRATCH_BYTES];

std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up on first use).
cudaError_t scratch_address(void** addr)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kMaxDevices)
        return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess)
            return e;
        g_scratch_addr[dev] = p;
    }
    *addr = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" ss_status selective_scan_fwd_noalloc(const ss_shape* shape, const void* u,
                                                const void* delta, const float* A, const void* B,
                                                const void* C, const float* Dskip, const void* z,
                                                const float* delta_bias, int32_t softplus,
                                                const ss_direction_map* dmap, void* out,
                                                float* last_state, void* stream,
                                                const ss_launch_opts* opts)
{
    size_t need = 0;
    ss_status st = selective_scan_workspace_size(shape, dmap, opts, &need);
    if (st != SS_OK)
        return st;
    if (need > SS_NOALLOC_SCRATCH_BYTES)
        return SS_ERR_SCRATCH_LIMIT;
    void* scratch = nullptr;
    if (need > 0 && scratch_address(&scratch) != cudaSuccess)
        return SS_ERR_CUDA;
    // Nothing in the scratch has to start at zero: every byte the kernels read from it was
    // written earlier in the same call.
    return selective_scan_fwd(shape, u, delta, A, B, C, Dskip, z, delta_bias, softplus, dmap, out,
                              last_state, need > 0 ? scratch : nullptr,
                              need > 0 ? SS_NOALLOC_SCRATCH_BYTES : 0, stream, opts);
}
