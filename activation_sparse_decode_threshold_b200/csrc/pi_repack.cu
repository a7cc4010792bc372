// pi_repack.cu -- load-time kernels that put a layer's weights into neuron-
// table order (PowerInfer (unite.ai), "Neuron placement and management": a
// table maps each stored neuron to its original position in the matrix).
//
//   repack_rows:  dst row p = src row perm[p] (optionally followed by the
//                 matching row of a second matrix, used to keep each INT4
//                 neuron's nibbles and scales in one contiguous record)
//   repack_bias:  dst[p] = src[perm[p]]
//   repack_down_transpose: W_down (d x F, output-major) -> neuron-major rows,
//                 row p = column perm[p]; tiled through shared memory, reading
//                 coalesced along the neuron axis and writing each output row
//                 segment contiguously (through the inverse table).
#include "pi_internal.h"

namespace pi {
namespace {

__global__ void k_repack_rows(const uint8_t *__restrict__ src, uint8_t *__restrict__ dst,
                              const int32_t *__restrict__ perm, int rows, int rb,
                              const uint8_t *__restrict__ src2, int rb2)
{
    const int p = blockIdx.x;
    if (p >= rows) return;
    const long long o = perm[p];
    const int out_rb = rb + rb2;
    const uint4 *s = reinterpret_cast<const uint4 *>(src + o * rb);
    uint4 *t = reinterpret_cast<uint4 *>(dst + (long long)p * out_rb);
    for (int i = threadIdx.x; i < rb / 16; i += blockDim.x) t[i] = s[i];
    if (src2) {
        const uint4 *s2 = reinterpret_cast<const uint4 *>(src2 + o * rb2);
        uint4 *t2 = reinterpret_cast<uint4 *>(dst + (long long)p * out_rb + rb);
        for (int i = threadIdx.x; i < rb2 / 16; i += blockDim.x) t2[i] = s2[i];
    }
}

__global__ void k_repack_bias(const float *__restrict__ src, float *__restrict__ dst,
                              const int32_t *__restrict__ perm, int n)
{
    const int p = blockIdx.x * blockDim.x + threadIdx.x;
    if (p < n) dst[p] = src[perm[p]];
}

template <typename T>
__global__ void k_down_transpose(const T *__restrict__ w, T *__restrict__ dst,
                                 const int32_t *__restrict__ inv, int d, int F)
{
    __shared__ T tile[32][33];
    const int i0 = blockIdx.x * 32, j0 = blockIdx.y * 32;
    const int tx = threadIdx.x, ty = threadIdx.y;   // 32 x 8
    for (int yy = ty; yy < 32; yy += 8) {
        const int j = j0 + yy, i = i0 + tx;
        if (j < d && i < F) tile[yy][tx] = w[(long long)j * F + i];
    }
    __syncthreads();
    for (int yy = ty; yy < 32; yy += 8) {
        const int i = i0 + yy, j = j0 + tx;
        if (i < F && j < d) dst[(long long)inv[i] * d + j] = tile[tx][yy];
    }
}

__global__ void k_invert(const int32_t *__restrict__ perm, int32_t *__restrict__ inv, int n)
{
    const int p = blockIdx.x * blockDim.x + threadIdx.x;
    if (p < n) inv[perm[p]] = p;
}

}  // namespace

cudaError_t repack_rows(const uint8_t *src, uint8_t *dst, const int32_t *perm, int rows,
                        int row_bytes, const uint8_t *src2, int row2_bytes, cudaStream_t s)
{
    if (rows <= 0) return cudaSuccess;
    k_repack_rows<<<rows, 128, 0, s>>>(src, dst, perm, rows, row_bytes, src2, src2 ? row2_bytes : 0);
    return cudaGetLastError();
}

cudaError_t repack_bias(const float *src, float *dst, const int32_t *perm, int n, cudaStream_t s)
{
    if (n <= 0) return cudaSuccess;
    k_repack_bias<<<(n + 255) / 256, 256, 0, s>>>(src, dst, perm, n);
    return cudaGetLastError();
}

// `perm` is the table (device).  The inverse table lives in a temporary
// stream-ordered allocation for the duration of the transpose (load time only).
cudaError_t repack_down_transpose(const uint8_t *w_down, uint8_t *dst, const int32_t *perm,
                                  int d, int F, int elem_bytes, cudaStream_t s)
{
    int32_t *inv = nullptr;
    cudaError_t e = cudaMallocAsync(&inv, sizeof(int32_t) * size_t(F), s);
    if (e != cudaSuccess) return e;
    k_invert<<<(F + 255) / 256, 256, 0, s>>>(perm, inv, F);
    dim3 grid((F + 31) / 32, (d + 31) / 32), block(32, 8);
    if (elem_bytes == 4)
        k_down_transpose<uint32_t><<<grid, block, 0, s>>>(
            reinterpret_cast<const uint32_t *>(w_down), reinterpret_cast<uint32_t *>(dst), inv, d, F);
    else
        k_down_transpose<uint16_t><<<grid, block, 0, s>>>(
            reinterpret_cast<const uint16_t *>(w_down), reinterpret_cast<uint16_t *>(dst), inv, d, F);
    e = cudaGetLastError();
    cudaError_t e2 = cudaFreeAsync(inv, s);
    return e != cudaSuccess ? e : e2;
}

}  // namespace pi
