// The bfloat16 scan kernel with bfloat16 delta, instantiated in a translation unit of its own so
// that the kernel variants compile in parallel.
#include "ss_fast.cuh"

namespace ss {

cudaError_t fast_launch_bf16(const ScanParams& p, int phase1, cudaStream_t stream, bool prepare_only)
{
    return fast_launch<__nv_bfloat16>(p, phase1, stream, prepare_only);
}

}  // namespace ss
