// Scan kernels instantiated for float io (a translation unit of its own so that the io types
// compile in parallel).
#include "ss_scan_kernels.cuh"

namespace ss {

cudaError_t launch_scan_f32(const ScanParams& p, int phase1, cudaStream_t stream)
{
    return launch_io<float>(p, phase1, stream);
}

}  // namespace ss
