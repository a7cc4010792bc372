// pi_decode_f16.cu -- decode kernels for weights F16 with predictor F16
// (one translation unit per format pair so the instantiations build in parallel).
#include "pi_decode_kernel.cuh"

namespace pi {

cudaError_t decode_launch_f16(int d, int mode, const DecodeParams &p, cudaStream_t st, bool query,
                                 int *blocks)
{
    return launch_fmt<kF16, kF16>(d, mode, p, st, query, blocks);
}

}  // namespace pi
