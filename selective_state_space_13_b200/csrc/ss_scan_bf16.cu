// Scan kernels instantiated for __nv_bfloat16 io (a translation unit of its own so that the io types
// compile in parallel).
#include "ss_scan_kernels.cuh"

namespace ss {

cudaError_t launch_scan_bf16(const ScanParams& p, int phase1, cudaStream_t stream)
{
    return launch_io<__nv_bfloat16>(p, phase1, stream);
}

}  // namespace ss
