// pi_decode_i4f16.cu -- decode kernels for weights I4 with predictor F16
// (one translation unit per format pair so the instantiations build in parallel).
#include "pi_decode_kernel.cuh"

namespace pi {

cudaError_t decode_launch_i4f16(int d, int mode, const DecodeParams &p, cudaStream_t st, bool query,
                                 int *blocks)
{
    return launch_fmt<kI4, kF16>(d, mode, p, st, query, blocks);
}

}  // namespace pi
