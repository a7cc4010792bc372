// pi_repack.cu -- load-time kernels that put a layer's weights into neuron-
// table order (PowerInfer (unite.ai), "Neuron placement and management": a
// table maps each stored neuron to its original position in the matrix).
//
//   repack_rows:  dst record p = row perm[p] of each source, concatenated
//                 (a neuron's gate and up rows, and for INT4 their nibbles
//                 and scales, become one contiguous record)
//   repack_bias:  dst[p] = src[perm[p]]
//   repack_down_transpose: W_down (d x F, output-major) -> neuron-major rows,
//                 row p = column perm[p]; tiled through shared memory, reading
//                 coalesced along the neuron axis and writing each output row
//                 segment contiguously (through the inverse table).
#include "pi_internal.h"

namespace pi {
namespace {

struct RepackSrc {
    const uint8_t *src[kMaxRepackSrc];
    int bytes[kMaxRepackSrc];
    int n;
};

__global__ void k_repack_rows(uint8_t *__restrict__ dst, const int32_t *__restrict__ perm, int rows,
                              RepackSrc rs, long long dst_stride)
{
    const int p = blockIdx.x;
    if (p >= rows) return;
    const long long o = perm[p];
    uint8_t *t = dst + (long long)p * dst_stride;
    for (int i = 0; i < rs.n; ++i) {
        const uint4 *s = reinterpret_cast<const uint4 *>(rs.src[i] + o * rs.bytes[i]);
        uint4 *tt = reinterpret_cast<uint4 *>(t);
        for (int j = threadIdx.x; j < rs.bytes[i] / 16; j += blockDim.x) tt[j] = s[j];
        t += rs.bytes[i];
    }
}

// Predictor U rows in table order with the 16-byte chunks of each row permuted
// inside every 128-byte group by the row's position in its strip modulo 8:
// chunk j goes to (j & ~7) | ((j ^ key) & 7), key = (p - strip start) & 7.
// Staged contiguously, the rows then let an 8-row matrix load hit eight
// different shared-memory bank groups.
__global__ void k_repack_u_swz(uint8_t *__restrict__ dst, const int32_t *__restrict__ perm, int rows,
                               const uint8_t *__restrict__ src, int row_bytes,
                               const int32_t *__restrict__ strip_off, int S)
{
    const int p = blockIdx.x;
    if (p >= rows) return;
    int lo = 0, hi = S - 1;                 // strip b with strip_off[b] <= p < strip_off[b + 1]
    while (lo < hi) {
        const int mid = (lo + hi + 1) / 2;
        if (strip_off[mid] <= p) lo = mid;
        else hi = mid - 1;
    }
    const int key = (p - strip_off[lo]) & 7;
    const uint4 *s = reinterpret_cast<const uint4 *>(src + (long long)perm[p] * row_bytes);
    uint4 *t = reinterpret_cast<uint4 *>(dst + (long long)p * row_bytes);
    for (int j = threadIdx.x; j < row_bytes / 16; j += blockDim.x) t[(j & ~7) | ((j ^ key) & 7)] = s[j];
}

__global__ void k_repack_bias(const float *__restrict__ src, float *__restrict__ dst,
                              const int32_t *__restrict__ perm, int n)
{
    const int p = blockIdx.x * blockDim.x + threadIdx.x;
    if (p < n) dst[p] = src[perm[p]];
}

template <typename T>
__global__ void k_down_transpose(const T *__restrict__ w, T *__restrict__ dst,
                                 const int32_t *__restrict__ inv, int d, int F, long long dst_stride)
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
        if (i < F && j < d) dst[(long long)inv[i] * dst_stride + j] = tile[tx][yy];
    }
}

__global__ void k_invert(const int32_t *__restrict__ perm, int32_t *__restrict__ inv, int n)
{
    const int p = blockIdx.x * blockDim.x + threadIdx.x;
    if (p < n) inv[perm[p]] = p;
}

// Records in table order -> the first hot_k of each strip to `hot` (index
// b * hot_k + loc) and the rest to `cold` (index p - (b + 1) * hot_k).
__global__ void k_split_records(const uint8_t *__restrict__ src, uint8_t *__restrict__ hot, uint8_t *__restrict__ cold,
                                int F, int bytes, const int32_t *__restrict__ strip_off, int S, int hot_k)
{
    const int p = blockIdx.x;
    if (p >= F) return;
    int lo = 0, hi = S - 1;                 // strip b with strip_off[b] <= p < strip_off[b + 1]
    while (lo < hi) {
        const int mid = (lo + hi + 1) / 2;
        if (strip_off[mid] <= p) lo = mid;
        else hi = mid - 1;
    }
    const int loc = p - strip_off[lo];
    uint8_t *dst = loc < hot_k ? hot + (size_t(lo) * hot_k + loc) * bytes
                               : cold + (size_t(p) - size_t(lo + 1) * hot_k) * bytes;
    const uint4 *s4 = reinterpret_cast<const uint4 *>(src + size_t(p) * bytes);
    for (int j = threadIdx.x; j < bytes / 16; j += blockDim.x) reinterpret_cast<uint4 *>(dst)[j] = s4[j];
}

}  // namespace

cudaError_t split_records(const uint8_t *src, uint8_t *hot, uint8_t *cold, int F, int bytes,
                          const int32_t *strip_off, int S, int hot_k, cudaStream_t s)
{
    if (F <= 0) return cudaSuccess;
    k_split_records<<<F, 128, 0, s>>>(src, hot, cold, F, bytes, strip_off, S, hot_k);
    return cudaGetLastError();
}

cudaError_t repack_rows(uint8_t *dst, const int32_t *perm, int rows, int n_src,
                        const uint8_t *const *src, const int *row_bytes, cudaStream_t s, long long dst_stride)
{
    if (rows <= 0) return cudaSuccess;
    if (n_src < 1 || n_src > kMaxRepackSrc) return cudaErrorInvalidValue;
    RepackSrc rs{};
    rs.n = n_src;
    for (int i = 0; i < n_src; ++i) {
        rs.src[i] = src[i];
        rs.bytes[i] = row_bytes[i];
    }
    long long packed = 0;
    for (int i = 0; i < n_src; ++i) packed += row_bytes[i];
    if (dst_stride == 0) dst_stride = packed;
    if (dst_stride < packed || dst_stride % 16 != 0) return cudaErrorInvalidValue;
    k_repack_rows<<<rows, 128, 0, s>>>(dst, perm, rows, rs, dst_stride);
    return cudaGetLastError();
}

cudaError_t repack_u_swizzled(uint8_t *dst, const int32_t *perm, int rows, const uint8_t *src, int row_bytes,
                              const int32_t *strip_off, int S, cudaStream_t s)
{
    if (rows <= 0) return cudaSuccess;
    if (row_bytes % 128 != 0) return cudaErrorInvalidValue;
    k_repack_u_swz<<<rows, 128, 0, s>>>(dst, perm, rows, src, row_bytes, strip_off, S);
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
                                  int d, int F, int elem_bytes, cudaStream_t s, long long dst_stride_bytes)
{
    if (dst_stride_bytes == 0) dst_stride_bytes = (long long)d * elem_bytes;
    if (dst_stride_bytes % elem_bytes != 0) return cudaErrorInvalidValue;
    const long long stride = dst_stride_bytes / elem_bytes;
    int32_t *inv = nullptr;
    cudaError_t e = cudaMallocAsync(&inv, sizeof(int32_t) * size_t(F), s);
    if (e != cudaSuccess) return e;
    k_invert<<<(F + 255) / 256, 256, 0, s>>>(perm, inv, F);
    dim3 grid((F + 31) / 32, (d + 31) / 32), block(32, 8);
    if (elem_bytes == 4)
        k_down_transpose<uint32_t><<<grid, block, 0, s>>>(
            reinterpret_cast<const uint32_t *>(w_down), reinterpret_cast<uint32_t *>(dst), inv, d, F, stride);
    else
        k_down_transpose<uint16_t><<<grid, block, 0, s>>>(
            reinterpret_cast<const uint16_t *>(w_down), reinterpret_cast<uint16_t *>(dst), inv, d, F, stride);
    e = cudaGetLastError();
    cudaError_t e2 = cudaFreeAsync(inv, s);
    return e != cudaSuccess ? e : e2;
}

}  // namespace pi
