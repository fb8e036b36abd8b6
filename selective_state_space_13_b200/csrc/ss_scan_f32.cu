// The scan kernel instantiated for float io (a translation unit of its own so that the kernel
// variants compile in parallel).
#include "ss_scan_kernels.cuh"

namespace ss {

cudaError_t scan_launch_f32(const ScanParams& p, int phase1, cudaStream_t stream, bool prepare_only)
{
    return launch_io<float>(p, phase1, stream, prepare_only);
}

}  // namespace ss
