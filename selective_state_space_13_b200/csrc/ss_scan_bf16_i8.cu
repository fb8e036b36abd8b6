// Scan kernels instantiated for bf16 io with int8 Delta codes (a translation unit of its own so
// that it compiles in parallel with the others).
#include "ss_scan_kernels.cuh"

namespace ss {

cudaError_t launch_scan_bf16_i8(const ScanParams& p, int phase1, cudaStream_t stream)
{
    return launch_io<__nv_bfloat16, int8_t>(p, phase1, stream);
}

}  // namespace ss
