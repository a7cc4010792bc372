// pi_decode_f16i8.cu -- decode kernels for weights F16 with the 8-bit per-row
// predictor (one translation unit per format pair so the instantiations build in parallel).
#include "pi_decode_kernel.cuh"

namespace pi {

cudaError_t decode_launch_f16i8(int d, int mode, const DecodeParams &p, cudaStream_t st, bool query,
                                 int *blocks)
{
    return launch_fmt<kF16, kI8>(d, mode, p, st, query, blocks);
}

}  // namespace pi
