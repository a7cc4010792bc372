// pi_decode.cu -- dispatch of the decode kernel (pi_decode_kernel.cuh) over
// weight / predictor formats, d_model class and layer kind.
#include "pi_internal.h"

namespace pi {

cudaError_t decode_launch_f32(int d, int mode, const DecodeParams &p, cudaStream_t st, bool query, int *blocks);
cudaError_t decode_launch_f16(int d, int mode, const DecodeParams &p, cudaStream_t st, bool query, int *blocks);
cudaError_t decode_launch_bf16(int d, int mode, const DecodeParams &p, cudaStream_t st, bool query, int *blocks);
cudaError_t decode_launch_i4f16(int d, int mode, const DecodeParams &p, cudaStream_t st, bool query, int *blocks);
cudaError_t decode_launch_i4bf16(int d, int mode, const DecodeParams &p, cudaStream_t st, bool query,
                                 int *blocks);
cudaError_t decode_launch_f16i8(int d, int mode, const DecodeParams &p, cudaStream_t st, bool query, int *blocks);
cudaError_t decode_launch_bf16i8(int d, int mode, const DecodeParams &p, cudaStream_t st, bool query, int *blocks);
cudaError_t decode_launch_i4i8(int d, int mode, const DecodeParams &p, cudaStream_t st, bool query, int *blocks);

namespace {

cudaError_t dispatch(int wfmt, int pfmt, int d, int mode, const DecodeParams &p, cudaStream_t st, bool query,
                     int *blocks)
{
    if (wfmt == kF32 && pfmt == kF32) return decode_launch_f32(d, mode, p, st, query, blocks);
    if (wfmt == kF16 && pfmt == kF16) return decode_launch_f16(d, mode, p, st, query, blocks);
    if (wfmt == kBF16 && pfmt == kBF16) return decode_launch_bf16(d, mode, p, st, query, blocks);
    if (wfmt == kI4 && pfmt == kF16) return decode_launch_i4f16(d, mode, p, st, query, blocks);
    if (wfmt == kI4 && pfmt == kBF16) return decode_launch_i4bf16(d, mode, p, st, query, blocks);
    if (wfmt == kF16 && pfmt == kI8) return decode_launch_f16i8(d, mode, p, st, query, blocks);
    if (wfmt == kBF16 && pfmt == kI8) return decode_launch_bf16i8(d, mode, p, st, query, blocks);
    if (wfmt == kI4 && pfmt == kI8) return decode_launch_i4i8(d, mode, p, st, query, blocks);
    return cudaErrorInvalidValue;
}

}  // namespace

int decode_mode(const DecodeParams &p)
{
    if (p.mode == kModePredict) return kModePred | (p.E > 1 ? kModeMoE : 0);
    return (p.E > 1 ? kModeMoE : 0) | (p.gated ? kModeGated : 0) | (p.spec_down ? kModeSpec : 0);
}

cudaError_t launch_decode(int wfmt, int pfmt, const DecodeParams &p, cudaStream_t stream)
{
    return dispatch(wfmt, pfmt, p.d, decode_mode(p), p, stream, false, nullptr);
}

int decode_max_blocks_per_sm(int wfmt, int pfmt, int d)
{
    // every instantiation has the same launch bounds and shared memory
    static const DecodeParams dummy{};
    int blocks = 0;
    if (dispatch(wfmt, pfmt, d, kModeGated | kModeSpec, dummy, nullptr, true, &blocks) != cudaSuccess) return 0;
    return blocks;
}

}  // namespace pi
