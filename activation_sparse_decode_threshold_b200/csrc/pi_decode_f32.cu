// pi_decode_f32.cu -- decode kernels for weights F32 with predictor F32
// (one translation unit per format pair so the instantiations build in parallel).
#include "pi_decode_kernel.cuh"

namespace pi {

cudaError_t decode_launch_f32(int d, int mode, const DecodeParams &p, cudaStream_t st, bool query,
                                 int *blocks)
{
    return launch_fmt<kF32, kF32>(d, mode, p, st, query, blocks);
}

}  // namespace pi
