// The bfloat16 scan kernel with int8 delta codes, instantiated in a translation unit of its own
// so that the kernel variants compile in parallel.
#include "ss_fast.cuh"

namespace ss {

cudaError_t fast_launch_bf16_i8(const ScanParams& p, int phase1, cudaStream_t stream,
                                bool prepare_only)
{
    return fast_launch<int8_t>(p, phase1, stream, prepare_only);
}

}  // namespace ss
