// The scan kernel instantiated for bfloat16 io (a translation unit of its own so that the kernel
// variants compile in parallel).
#include "ss_scan_kernels.cuh"

namespace ss {

cudaError_t scan_launch_bf16(const ScanParams& p, int phase1, cudaStream_t stream, bool prepare_only)
{
    return launch_io<__nv_bfloat16>(p, phase1, stream, prepare_only);
}

}  // namespace ss
