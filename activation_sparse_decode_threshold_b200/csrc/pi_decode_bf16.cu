// pi_decode_bf16.cu -- decode kernels for weights BF16 with predictor BF16
// (one translation unit per format pair so the instantiations build in parallel).
#include "pi_decode_kernel.cuh"

namespace pi {

cudaError_t decode_launch_bf16(int d, int mode, const DecodeParams &p, cudaStream_t st, bool query,
                                 int *blocks)
{
    return launch_fmt<kBF16, kBF16>(d, mode, p, st, query, blocks);
}

}  // namespace pi
