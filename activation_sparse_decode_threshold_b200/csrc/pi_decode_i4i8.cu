// pi_decode_i4i8.cu -- decode kernels for weights INT4G32 with the 8-bit per-row
// predictor (one translation unit per format pair so the instantiations build in parallel).
#include "pi_decode_kernel.cuh"

namespace pi {

cudaError_t decode_launch_i4i8(int d, int mode, const DecodeParams &p, cudaStream_t st, bool query,
                                 int *blocks)
{
    return launch_fmt<kI4, kI8>(d, mode, p, st, query, blocks);
}

}  // namespace pi
