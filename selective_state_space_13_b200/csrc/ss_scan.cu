// Host side of the scan kernels: the launch dispatch over io types, the direction merge, the
// index map for the host, and the device error word that bounded waits report to.
#include <cuda_runtime.h>

#include <mutex>

#include "ss_scan_kernels.cuh"

namespace ss {

// Set (bitwise or) by any CTA whose bounded wait gave up; read and cleared by read_status.
__device__ unsigned int g_ss_status = 0;

namespace {
std::mutex g_status_mutex;
constexpr int kMaxDevices = 64;
unsigned int* g_status_addr[kMaxDevices] = {};
}  // namespace

unsigned int* status_word()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return nullptr;
    std::lock_guard<std::mutex> lock(g_status_mutex);
    if (!g_status_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_ss_status) != cudaSuccess)
            return nullptr;
        g_status_addr[dev] = static_cast<unsigned int*>(p);
    }
    return g_status_addr[dev];
}

int channels_per_cta() { return 32 * kWarps; }

namespace {

cudaError_t launch_any(const ScanParams& p, int io_dtype, int phase1, cudaStream_t stream,
                       bool prepare_only)
{
    if (io_dtype == SS_BF16)
        return p.delta_scale ? scan_launch_bf16_i8(p, phase1, stream, prepare_only)
                             : scan_launch_bf16(p, phase1, stream, prepare_only);
    return scan_launch_f32(p, phase1, stream, prepare_only);
}

}  // namespace

cudaError_t prepare_scan(ScanParams& p, int io_dtype)
{
    cudaError_t e;
    if (io_dtype == SS_BF16)
        e = p.delta_scale ? make_maps<__nv_bfloat16, int8_t>(p, p.z != nullptr, 32 * kWarps)
                          : make_maps<__nv_bfloat16, __nv_bfloat16>(p, p.z != nullptr, 32 * kWarps);
    else
        e = make_maps<float, float>(p, p.z != nullptr, 32 * kWarps);
    if (e != cudaSuccess)
        return e;
    if (p.S > 1 && (e = launch_any(p, io_dtype, 1, nullptr, true)) != cudaSuccess)
        return e;
    return launch_any(p, io_dtype, 0, nullptr, true);
}

cudaError_t launch_scan(const ScanParams& p, int io_dtype, int phase1, cudaStream_t stream)
{
    return launch_any(p, io_dtype, phase1, stream, false);
}

template <typename io_t, bool GATE>
cudaError_t merge_k(const MergeParams& p, unsigned blocks, cudaStream_t stream)
{
    // the merge may launch before the scan ends; it waits for the scan's outputs itself
    switch (p.K) {
    case 2: return launch_ex(merge_kernel<io_t, GATE, 2>, blocks, 256, 0, stream, true, p);
    case 3: return launch_ex(merge_kernel<io_t, GATE, 3>, blocks, 256, 0, stream, true, p);
    default: return launch_ex(merge_kernel<io_t, GATE, 4>, blocks, 256, 0, stream, true, p);
    }
}

cudaError_t launch_merge(const MergeParams& p, int io_dtype, cudaStream_t stream)
{
    const int64_t n4 = p.rows * p.D / 4;
    if (n4 <= 0)
        return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t blocks = (n4 + 255) / 256;
    if (blocks > static_cast<int64_t>(sms) * 8)
        blocks = static_cast<int64_t>(sms) * 8;
    const unsigned nb = static_cast<unsigned>(blocks);
    const bool gate = p.z != nullptr;
    if (io_dtype == SS_BF16)
        return gate ? merge_k<__nv_bfloat16, true>(p, nb, stream)
                    : merge_k<__nv_bfloat16, false>(p, nb, stream);
    return gate ? merge_k<float, true>(p, nb, stream) : merge_k<float, false>(p, nb, stream);
}

int64_t position_host(int32_t dir, int64_t L, int32_t H, int32_t W, int64_t t)
{
    return position(dir, L, H, W, t);
}

cudaError_t read_status(cudaStream_t stream, bool clear, unsigned int* value)
{
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess)
        return e;
    e = cudaMemcpyFromSymbol(value, g_ss_status, sizeof(unsigned int));
    if (e != cudaSuccess || !clear)
        return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_ss_status, &zero, sizeof(unsigned int));
}

}  // namespace ss
