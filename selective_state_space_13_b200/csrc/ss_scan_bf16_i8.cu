// The scan kernel instantiated for bfloat16 io with int8 delta codes (a translation unit of its
// own so that it compiles in parallel with the others).
#include "ss_scan_kernels.cuh"

namespace ss {

cudaError_t scan_launch_bf16_i8(const ScanParams& p, int phase1, cudaStream_t stream,
                                bool prepare_only)
{
    return launch_io<__nv_bfloat16, int8_t>(p, phase1, stream, prepare_only);
}

}  // namespace ss
