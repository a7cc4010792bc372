// pi_decode_kernel.cuh -- persistent sparse-FFN decode kernel for sm_100a.
//
// One cooperative launch runs a range of layers for one token.  Each CTA owns
// one strip of the neuron table (a contiguous run of table positions holding
// a balanced share of hot neurons, hottest first), a few rows of t and one
// slice of the d_model columns.  Per layer l (dense FFN):
//
//   [B] z = U t - c over the strip (tensor-core dots of the staged U rows),
//       active iff z > threshold, the active list compacted in ascending
//       table order with warp ballots (PowerInfer (unite.ai), "Adaptive
//       sparse predictor").
//   [balance] every strip publishes its active list; after a grid barrier
//       each CTA takes an equal share of the lists concatenated in strip
//       order (depends only on the active set: deterministic).
//   [C] for the active neurons of its share: the neuron's record (W_gate /
//       W_up rows, plus its W_down row for ReLU / ReGLU, where h != 0 almost
//       always follows z > 0) by bulk copy into shared memory -> h =
//       act(g, u) (INT4 records: dots on the integer tensor cores with x as
//       base-128 digits); for h != 0 its W_down column (stored as a row)
//       accumulates into a per-CTA fp32 partial of y ("Neuron-aware
//       operators": rows of the input matrices, columns of the output matrix).
//   [merge] each CTA's partial, rounded to 64-bit fixed point, is added into
//       the layer's total by one bulk reduction in L2 (integer adds: the total
//       does not depend on arrival order; the merge of partial results,
//       nearauto.com PowerInfer article, Fig. 8).
//   --- grid barrier ---
//   [next input] every CTA reads the whole total and forms the whole next
//       input r + y, its sum of squares and x = RMSNorm(r + y) in the same
//       order (so every CTA holds the same x); its columns of r + y go to the
//       next input buffer, its own rows of t = V x for layer l + 1 to every
//       CTA as tagged 64-bit slots (value and layer tag in one store), which
//       the next layer's start polls instead of a grid barrier.
//
// Two grid barriers per layer.  A routed (MoE) layer adds each CTA's column
// share of the router logits into 64-bit fixed-point totals in the [next
// input] step, passes a third grid barrier, picks its two experts the same
// way in every CTA, and takes its rows of t from the chosen experts' V.
//
// Memory: weight bytes are pulled towards the SM as soon as their addresses
// are known.  A strip's active records are prefetched into L2 the moment its
// list is published; the next layer's V rows of this CTA and biases (router
// rows when routed) are prefetched into L2 when the gather starts; when it
// ends, they are bulk-copied into shared memory with the first rows of the
// next U strip, and land during the merge and its barrier.  All waits are
// bounded (%globaltimer); a wait that runs out records an error word and
// every CTA returns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#pragma once
#include "pi_internal.h"

namespace pi {
namespace {

// ---------------------------------------------------------------------------
// PTX helpers
// ---------------------------------------------------------------------------
// Bulk prefetch of a global range into L2 (fire and forget), 32 KB pieces.
__device__ __forceinline__ void prefetch_l2(const void *src, uint32_t bytes)
{
    const uint8_t *p = static_cast<const uint8_t *>(src);
    for (uint32_t o = 0; o < bytes; o += 32768u) {
        const uint32_t n = bytes - o < 32768u ? bytes - o : 32768u;
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p + o), "r"(n) : "memory");
    }
}
// Read-only weight loads that do not allocate in L1.
__device__ __forceinline__ uint4 ldw4(const uint8_t *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}
__device__ __forceinline__ uint32_t ldw1(const uint8_t *p)
{
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ uint2 ldw2(const uint8_t *p)
{
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}
__device__ __forceinline__ uint32_t s2u(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t *b, unsigned count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(s2u(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint64_t *b, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(s2u(b)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *b, uint32_t bytes)
{
    asm volatile("mbarrier.expect_tx.shared::cta.b64 [%0], %1;" ::"r"(s2u(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *b)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(s2u(b)) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t *b, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(s2u(b)), "r"(parity)
        : "memory");
    return ok != 0;
}
// 1-D bulk copy global -> this CTA's shared memory, completion on `bar`.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(s2u(dst)), "l"(src), "r"(bytes), "r"(s2u(bar))
        : "memory");
}
__device__ __forceinline__ long long gtimer()
{
    long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void cta_sync()
{
    asm volatile("bar.sync 0;" ::: "memory");
}
__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned *p)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// Tagged 64-bit slots: one strong 64-bit access moves a 32-bit value and its
// tag together, so a reader that sees the tag it expects also sees the value.
__device__ __forceinline__ void st_relaxed_u64(unsigned long long *p, unsigned long long v)
{
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long *p)
{
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void red_add_u64(unsigned long long *p, unsigned long long v)
{
    asm volatile("red.relaxed.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ void red_release_gpu(unsigned *p, unsigned v)
{
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_vol(const int *p)
{
    return *reinterpret_cast<const volatile int *>(p);
}
__device__ __forceinline__ void st_vol(int *p, int v)
{
    *reinterpret_cast<volatile int *>(p) = v;
}

// ---------------------------------------------------------------------------
// Stored formats.  A vector is 16 bytes of a row (4 bytes for INT4: 8
// nibbles, a quarter of a 32-element scale group; 8 bytes for INT8).
// ---------------------------------------------------------------------------
template <int F> struct Fm;
template <> struct Fm<kF32>  { static constexpr int VB = 16, EPV = 4;  using V = uint4; };
template <> struct Fm<kF16>  { static constexpr int VB = 16, EPV = 8;  using V = uint4; };
template <> struct Fm<kBF16> { static constexpr int VB = 16, EPV = 8;  using V = uint4; };
template <> struct Fm<kI4>   { static constexpr int VB = 4,  EPV = 8;  using V = uint32_t; };   // 8 nibbles
template <> struct Fm<kI8>   { static constexpr int VB = 8,  EPV = 8;  using V = uint2; };   // signed bytes (row scale apart)

template <int F>
__device__ __forceinline__ typename Fm<F>::V ldvec(const uint8_t *p)
{
    if constexpr (F == kI4) return ldw1(p);
    else if constexpr (F == kI8) return ldw2(p);
    else return ldw4(p);
}

template <int F>
__device__ __forceinline__ void cvt(const typename Fm<F>::V &v, float *o)
{
    if constexpr (F == kF32) {
        o[0] = __uint_as_float(v.x); o[1] = __uint_as_float(v.y);
        o[2] = __uint_as_float(v.z); o[3] = __uint_as_float(v.w);
    } else if constexpr (F == kF16) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[i]));
            o[2 * i] = f.x;
            o[2 * i + 1] = f.y;
        }
    } else if constexpr (F == kBF16) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            o[2 * i] = __uint_as_float(w[i] << 16);
            o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    } else if constexpr (F == kI8) {
        const uint32_t w[2] = {v.x, v.y};
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) o[4 * i + j] = float(int8_t(uint8_t(w[i] >> (8 * j))));
    } else {
        // element 2j sits in the low nibble of byte j; n - 8 is formed exactly
        // by placing n in the mantissa of 2^23 and subtracting 2^23 + 8
#pragma unroll
        for (int j = 0; j < 8; ++j) o[j] = __uint_as_float(0x4b000000u | ((v >> (4 * j)) & 0xfu)) - 8388616.0f;
    }
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Warp reduction of N values per lane (N a power of two <= 32): after it,
// lane L holds the warp-wide sum of value L / (32 / N).  At each of the first
// log2(N) stages a lane keeps one half of its values, chosen by its lane bit,
// and adds the partner's copy of that half; the lanes left sharing a value
// finish with a plain butterfly.  N - 1 + log2(32 / N) shuffles.
template <int N>
__device__ __forceinline__ float warp_transpose_sum(float (&v)[N])
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 16, n = N; n > 1; o >>= 1, n >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < n / 2; ++i) {
            const float send = upper ? v[i] : v[i + n / 2];
            const float keep = upper ? v[i + n / 2] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
#pragma unroll
    for (int o = 32 / N / 2; o >= 1; o >>= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    return v[0];
}

// Four 8x8 b16 matrices from shared memory (lane L gives the address of row
// L % 8 of matrix L / 8).
__device__ __forceinline__ void ldsm_x4(const void *p, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(s2u(p)));
}
__device__ __forceinline__ void ldsm_x4_a(uint32_t saddr, uint32_t (&r)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(saddr));
}
// D += A (16x16, row) * B (16x8, col), 16-bit inputs of format F, fp32 accumulate.
template <int F>
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1)
{
    if constexpr (F == kBF16)
        asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                     "{%8, %9}, {%0, %1, %2, %3};"
                     : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                     : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    else
        asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                     "{%8, %9}, {%0, %1, %2, %3};"
                     : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
                     : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// An fp32 value as an unevaluated sum of 16-bit values of format F: two fp16
// parts (22 significant bits) or up to three bf16 parts (24 bits; two, 16
// bits, where shared memory holds only two per value).  Multiplying a 16-bit
// weight by each part is exact in fp32, so a tensor-core dot with the parts as
// columns of B, summed over the columns, carries the fp32 operand rather than
// a 16-bit rounding of it.  Part p of value k is written at out[p * stride + k].
template <int F>
__device__ __forceinline__ void split_parts(float x, int nparts, uint16_t *out, int stride)
{
    if constexpr (F == kBF16) {
        const __nv_bfloat16 h = __float2bfloat16_rn(x);
        const float r1 = x - __bfloat162float(h);
        const __nv_bfloat16 m = __float2bfloat16_rn(r1);
        out[0] = __bfloat16_as_ushort(h);
        out[stride] = __bfloat16_as_ushort(m);
        if (nparts > 2) out[2 * stride] = __bfloat16_as_ushort(__float2bfloat16_rn(r1 - __bfloat162float(m)));
    } else {
        const __half h = __float2half_rn(x);
        out[0] = __half_as_ushort(h);
        out[stride] = __half_as_ushort(__float2half_rn(x - __half2float(h)));
    }
}

// Eight INT4 codes (nibble i of w = element i, code n_i, value n_i - 8) as
// signed bytes 16 (n_i - 8), exactly: flipping a nibble's top bit gives the
// value in 4-bit two's complement, and moving it to the top of a byte scales
// it by 16.  ev holds elements 0, 2, 4, 6 (byte j = element 2j), od holds
// elements 1, 3, 5, 7.
__device__ __forceinline__ void i4x8_to_s8(uint32_t w, uint32_t &ev, uint32_t &od)
{
    ev = ((w << 4) ^ 0x80808080u) & 0xf0f0f0f0u;
    od = (w ^ 0x80808080u) & 0xf0f0f0f0u;
}
// D = A B of signed bytes, 32-bit integer result (exact), C = 0.
__device__ __forceinline__ void imma16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                 "{%8, %9}, {%10, %10, %10, %10};"
                 : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(0));
}
// D += A B of signed bytes, 32-bit integer accumulators (exact).
__device__ __forceinline__ void imma16832_acc(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                 "{%8, %9}, {%0, %1, %2, %3};"
                 : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// An integer of magnitude below 2^22 as fp32, exactly: placed in the mantissa
// of 1.5 * 2^23, which is then subtracted.
__device__ __forceinline__ float i22_to_f(int c)
{
    return __int_as_float(c + 0x4B400000) - 12582912.0f;
}

// Where a neuron's record lives.  Without a VRAM budget (hot_k = 0) every
// record is in HBM at its table position.  With one, the first hot_k
// positions of each strip stay in HBM, packed strip by strip (index
// b * hot_k + loc), and the others live in pinned host memory, packed in
// table order (index pos - (b + 1) * hot_k).  The code is the index, with bit
// 23 set for a record in host memory.
constexpr unsigned kColdBit = 1u << 23;
__device__ __forceinline__ unsigned rec_code(int hot_k, int b, int loc, int pos)
{
    if (hot_k == 0) return unsigned(pos);
    if (loc < hot_k) return unsigned(b * hot_k + loc);
    return kColdBit | unsigned(pos - (b + 1) * hot_k);
}
// 16-byte pieces [lo, hi) of a record in host memory into shared memory, by
// the calling threads (plain loads: the bytes cross the host link)
__device__ __forceinline__ void copy_host_rec(uint8_t *dst, const uint8_t *src, int bytes, int t0, int nt)
{
    for (int i = t0; i < bytes / 16; i += nt)
        reinterpret_cast<uint4 *>(dst)[i] = *reinterpret_cast<const uint4 *>(src + 16 * size_t(i));
}

__device__ __forceinline__ float act_h(int act, float g, float u)
{
    const float gp = g > 0.f ? g : 0.f;
    if (act == 0) return gp;               // ReLU (non-gated)
    if (act == 1) return gp * u;           // ReGLU
    return gp * (u > 0.f ? u : 0.f);       // dReLU
}

constexpr int kRA = 16;           // V rows per staging round at most
constexpr int kZRows = 112;       // U rows per staging round at most (a multiple of 16)
constexpr int kMaxU = 4;          // U vectors per lane (rank <= 128 * EPV)
constexpr int kRound = 20;        // neurons per gather round at most (a routed strip share of ~19 in one round)
constexpr int kIssue = 32;        // neurons whose records are in flight at once at most
static_assert(kRound <= 32, "a round's neurons are tracked in one warp ballot");
constexpr int kRed = 2 * kRound;  // values reduced per warp at most

struct Smem {
    float red[2][kConsumerWarps][kRed];
    union {
        float zred[kConsumerWarps][kZRows];    // per-warp partial logits of a U round (logit phase)
        struct {                               // this CTA's share of the active list (gather phase)
            int32_t glst[kMaxTopK * kMaxStrip];  // (slot << 24) | table position
            float gc[kMaxTopK * kMaxStrip];      // their biases
        };
        ExpertDev exall[kMaxExperts];          // every expert's weight pointers (MoE layer start)
    };
    int scan[kMaxStrips + 1];              // exclusive prefix of the strip counts
    union {                                // layer start .. logits / gather
        alignas(16) float tsm[kMaxRankTotal];  // t (fp32 predictor) or its 16-bit parts (split_parts)
        struct {
            int32_t nz[kMaxTopK * kMaxStrip];  // neurons with h != 0, encoded as glst
            float hz[kMaxTopK * kMaxStrip];    // their h (routing weight folded in)
        };
    };
    union {                                // input forming / layer start .. active list
        alignas(16) float rsl[kMaxSliceCols];  // this CTA's columns of the new residual
        struct {
            float cbuf[kMaxTopK][kMaxStrip];
            float zbuf[kMaxTopK][kMaxStrip];
        };
    };
    ExpertDev exl[2][kMaxTopK];            // weight pointers of the layer's expert slots, by layer parity
    int16_t lst[kMaxTopK * kMaxStrip];     // active neurons: (slot << 12) | local
    int lst_n[kMaxTopK];
    int share_n;                           // size of this CTA's share of the active list
    float rsum[kRed];                      // CTA-wide dot products of a gather round
    float rh[kRound];                      // h of each neuron of a gather round
    int route_e[kMaxTopK];
    float route_w[kMaxTopK];
    int bc[2];
    uint64_t stage_bar;                    // completion of a staging round
    uint64_t vbar;                         // completion of the next layer's V rows (dense), staged after the y arrival
    uint64_t gbar[kIssue / 4];             // completion of each group of four neurons of a gather batch
    int gfail;                             // a warp's bounded wait on a group ran out
};

__device__ void set_error(int *err, int code)
{
    atomicCAS(err, 0, code);
}

__device__ __forceinline__ void prof_put(const DecodeParams &p, int li, int point, long long v)
{
    if (p.prof && threadIdx.x == 0)
        p.prof[(size_t(li) * kProfPoints + point) * gridDim.x + blockIdx.x] = v;
}

// Fixed-point accumulation (exact, so the result does not depend on the
// order in which CTAs arrive): values are rounded to multiples of 2^-32 and
// added as 64-bit integers.  A scaled value of magnitude 2^55 or more (or not
// finite) could make the sum over up to 256 CTAs leave the int64 range: it is
// recorded as a failed device check (the caller's pi_sync reports
// PI_ERR_DEVICE_CHECK) instead of wrapping silently.
constexpr float kFixT = 4294967296.0f;    // 2^32
constexpr float kFixMax = 36028797018963968.0f;   // 2^55
__device__ __forceinline__ unsigned long long fix_q(float v, int *err)
{
    const float sv = v * kFixT;
    if (!(fabsf(sv) < kFixMax)) {
        set_error(err, kDevCheck);
        return 0ull;
    }
    return static_cast<unsigned long long>(__float2ll_rn(sv));
}

// Shared-memory writes made visible to the bulk-copy (async) proxy, and the
// executing thread's generic and async views of global memory ordered.
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_global()
{
    asm volatile("fence.proxy.async.global;" ::: "memory");
}
// dst[i] += src[i] for `bytes` of 64-bit integers, by bulk reductions from
// this CTA's shared memory (32 KB pieces), committed as one bulk group.
__device__ __forceinline__ void bulk_reduce_add_u64(unsigned long long *dst, const void *src, uint32_t bytes)
{
    for (uint32_t o = 0; o < bytes; o += 32768u) {
        const uint32_t n = bytes - o < 32768u ? bytes - o : 32768u;
        asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.u64 [%0], [%1], %2;"
                     ::"l"(reinterpret_cast<uint8_t *>(dst) + o), "r"(s2u(src) + o), "r"(n)
                     : "memory");
    }
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until this thread's bulk groups have completed (their writes performed).
__device__ __forceinline__ void bulk_wait_all()
{
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Grid-wide barrier of all CTAs of the cooperative launch, in two halves so
// that a CTA can issue work between its arrival and its wait.  Thread 0
// arrives with a release on one counter (after the block barrier, so it
// carries the whole CTA's writes) and then polls it with acquires until all
// S CTAs of this barrier's epoch have arrived, bounded by wait_ns; the
// verdict is broadcast through shared memory so the whole CTA agrees.  The
// counter is never reset within a launch.  (Measured on the B200: one counter
// polled by one thread per CTA completes a barrier of 148 CTAs in about 1.3
// us, against 1.7 us for arrivals spread over 16 counters polled by a warp.)
__device__ __forceinline__ void grid_arrive(const DecodeParams &p, unsigned &epoch)
{
    cta_sync();
    epoch += 1;
    if (threadIdx.x == 0) red_release_gpu(p.bar, 1u);
}
__device__ bool grid_wait(Smem *sm, const DecodeParams &p, unsigned epoch, int &bci, long long *cyc)
{
    if (threadIdx.x == 0) {
        const long long c0 = clock64();
        unsigned target = epoch * gridDim.x;
        if ((p.debug_flags & 1) && epoch == 1) target += 1;   // PI_DEBUG_STALL_BARRIER
        bool ok = true;
        if (ld_acquire_gpu(p.bar) < target) {
            const long long t0 = gtimer();
            for (unsigned it = 1;; ++it) {
                if (ld_acquire_gpu(p.bar) >= target) break;
                if ((it & 31) == 0 && gtimer() - t0 > p.wait_ns) {
                    set_error(p.err, kDevTimeout);
                    ok = false;
                    break;
                }
            }
        }
        st_vol(&sm->bc[bci], ok ? 1 : 0);
        if (cyc) *cyc += clock64() - c0;
    }
    cta_sync();
    const bool ok = ld_vol(&sm->bc[bci]) != 0;
    bci ^= 1;
    return ok;
}
__device__ __forceinline__ bool grid_sync(Smem *sm, const DecodeParams &p, unsigned &epoch, int &bci, long long *cyc)
{
    grid_arrive(p, epoch);
    return grid_wait(sm, p, epoch, bci, cyc);
}

// Staging round: thread 0 has issued bulk copies onto sm->stage_bar (or
// `bar`); it waits (bounded) and the whole CTA adopts its verdict.
__device__ bool stage_wait(Smem *sm, const DecodeParams &p, uint32_t &par, int &bci,
                           long long *cyc = nullptr, uint64_t *bar = nullptr)
{
    if (!bar) bar = &sm->stage_bar;
    if (threadIdx.x == 0) {
        const long long c0 = clock64();
        bool ok = mbar_test(bar, par);
        if (!ok) {
            const long long t0 = gtimer();
            for (unsigned it = 1; !ok; ++it) {
                ok = mbar_test(bar, par);
                if (!ok && (it & 15) == 0 && gtimer() - t0 > p.wait_ns) {
                    set_error(p.err, kDevTimeout);
                    break;
                }
            }
        }
        st_vol(&sm->bc[bci], ok ? 1 : 0);
        if (cyc) *cyc += clock64() - c0;
    }
    cta_sync();
    const bool ok = ld_vol(&sm->bc[bci]) != 0;
    bci ^= 1;
    if (ok) {
        mbar_test(bar, par);   // acquire for this thread (phase complete)
        par ^= 1;                         // a failed round keeps its phase for the drain
    }
    return ok;
}

// Issue bulk copies of [src, src + bytes) into dst in pieces of <= 32 KB.
__device__ __forceinline__ void stage_copy(uint8_t *dst, const uint8_t *src, uint32_t bytes, uint64_t *bar)
{
    for (uint32_t o = 0; o < bytes; o += 32768u) {
        const uint32_t n = bytes - o < 32768u ? bytes - o : 32768u;
        bulk_g2s(dst + o, src + o, n, bar);
    }
}

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------
template <int WF, int PF, int DMAX, int MODE>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ DecodeParams p)
{
    constexpr int EPVW = Fm<WF>::EPV, EPVP = Fm<PF>::EPV, VBW = Fm<WF>::VB, VBP = Fm<PF>::VB;
    constexpr int MAXVW = (DMAX / EPVW + kThreads - 1) / kThreads;
    using VW = typename Fm<WF>::V;
    using VP = typename Fm<PF>::V;

    __shared__ Smem sm;
    extern __shared__ __align__(128) uint8_t stg[];   // kStageBytes staging buffer
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.x, S = gridDim.x;
    const int d = p.d, r = p.r;
    const int s0 = p.strip_off[b], ns = p.strip_off[b + 1] - s0;
    // layer kind, fixed per instantiation so each kernel holds only its path
    constexpr bool moe = (MODE & kModeMoE) != 0;
    constexpr bool kGated = (MODE & kModeGated) != 0;
    constexpr bool kSpec = (MODE & kModeSpec) != 0;
    constexpr bool predict = (MODE & kModePred) != 0;   // pi_predict: one layer, stop after the list
    const int ntop = predict ? 1 : p.top_k;
    const int nvecW = (WF == kI4 ? d / 2 : d * (WF == kF32 ? 4 : 2)) / VBW;
    const int nvecU = p.urow / VBP;
    const int l0 = p.layer_begin;
    const int l1 = predict ? p.layer_begin + 1 : p.layer_end;
    // this CTA's columns of the residual (8-column groups)
    const int c0 = 8 * p.grp_off[b], ncol = 8 * (p.grp_off[b + 1] - p.grp_off[b]);
    // this CTA's rows of t (rows [a0, a1) of the layer's experts' ranks together)
    const int rows_total = ntop * r;
    const int a0 = int((long long)b * rows_total / S), a1 = int((long long)(b + 1) * rows_total / S);
    const int nrows = a1 - a0;
    // U rows per staging round: the whole strip when it fits, else rounds of a
    // multiple of 8 rows (chunk permutation keys are row mod 8)
    const int ucap_rows = min(kZRows, kStageBytes / p.urow);
    const int ucap = ns <= ucap_rows ? max(ns, 1) : (ucap_rows & ~7);
    // routed: when both experts' strips fit the staging buffer together (an
    // 8-bit predictor's rows), both are staged right after this CTA's rows
    // of t, the second right after the first (chunk permutation keys are
    // relative to each strip's own first row)
    const int u2 = ns;
    const bool both_u = moe && !predict && p.top_k == 2 && ns > 0 && ns <= ucap && 2 * ns * p.urow <= kStageBytes;

    // Staging buffer at the end of a layer (decode): this CTA's partial of y
    // as fixed-point values at the top [yoff, end); below it the next layer's
    // V rows of this CTA [voff, yoff) (dense, when they fit: issued when the
    // gather ends, they land during the reduction and its barrier); below
    // them the first `ufirst` rows of the next U strip's first round, whose
    // other rows follow once the V rows have been read.  A routed layer
    // stages its V rows in rounds from offset 0 once the experts are known.
    const int yoff = predict ? kStageBytes : kStageBytes - d * 8;
    // INT4 weights: x as signed base-128 digits in the tensor-core B layout of
    // the gather's dots (8d bytes at the top of the staging buffer, written
    // after the predictor's rounds and read until the last gather round).
    // |x_j| <= sqrt(d) after the RMSNorm, so x * xs with xs = 2^(6 - e),
    // 4^e >= d, lies in [-64, 64]; digit 0 is its nearest integer and each
    // further digit the nearest integer of 128 times the remainder, so that
    // x = xs^-1 sum_{p<5} digit_p 128^-p up to 2^-29 xs^-1, every step exact.
    const int xpoff = kStageBytes - 8 * d;
    const uint8_t *xp = stg + xpoff;
    int xse = 0;
    while ((1 << (2 * xse)) < d) ++xse;
    const float xs = ldexpf(1.f, 6 - xse);
    const int voff = (yoff - nrows * p.vrow) & ~127;
    const bool vsm = !moe && nrows > 0 && nrows <= kRA && voff >= 0;
    const int u_round0 = min(ns, ucap);
    const int ufirst = vsm ? min(u_round0, voff / p.urow) : u_round0;

    float tsc = 1.f;   // 8-bit predictor: the scale of t's digits in this layer
    // the rows of t as tagged slots (tag: the layer's index in this launch + 1)
    unsigned long long *const tslot = reinterpret_cast<unsigned long long *>(p.bar + kTagTWord);
    unsigned epoch = 0;
    uint32_t spar = 0;
    uint32_t gpar = 0, gpend = 0;   // gather group barriers: phase parities, groups in flight
    int bci = 0, rb = 0;
    bool staged_early = false;   // round 0 of the next U strip is already in flight
    bool pending = false;        // a staging round was issued and not yet waited for
    uint32_t vpar = 0;
    bool vpend = false;          // V rows (dense) issued on vbar, not yet waited for
    bool upart2 = false;         // the staged U round still misses its second piece

    // stage rows [row0, row0 + n) of an expert's U strip, contiguous, at
    // staged row `at` (lane 0 of warp 0 issues the copies); a round staged in
    // two pieces announces the first piece's bytes without arriving, and its
    // second piece arrives (`last`)
    auto stage_u_at = [&](const ExpertDev &ex, int row0, int n, int at, bool last) {
        if (lane == 0) {
            if (last) mbar_arrive_tx(&sm.stage_bar, uint32_t(n) * p.urow);
            else mbar_expect_tx(&sm.stage_bar, uint32_t(n) * p.urow);
            if (n > 0)
                stage_copy(stg + size_t(at) * p.urow, ex.U + size_t(s0 + row0) * p.urow, uint32_t(n) * p.urow,
                           &sm.stage_bar);
        }
    };
    auto stage_u = [&](const ExpertDev &ex, int row0, int n) { stage_u_at(ex, row0, n, 0, true); };
    // dense, warp 0: layer ln's V rows of this CTA onto vbar and the first
    // piece of its first U round onto stage_bar (the rest of the strip into L2)
    auto stage_next_dense = [&](int ln) {
        const ExpertDev &nx = sm.exl[ln & 1][0];
        if (lane == 0) {
            mbar_arrive_tx(&sm.vbar, uint32_t(nrows) * p.vrow);
            stage_copy(stg + voff, nx.V + size_t(a0) * p.vrow, uint32_t(nrows) * p.vrow, &sm.vbar);
        }
        if (ns > 0) {
            stage_u_at(nx, 0, ufirst, 0, ufirst == u_round0);
            if (lane == 0 && ns > ucap)
                prefetch_l2(nx.U + size_t(s0 + ucap) * p.urow, uint32_t(ns - ucap) * p.urow);
        }
    };

    if (tid == 0) {
        mbar_init(&sm.stage_bar, 1);
        mbar_init(&sm.vbar, 1);
        for (int g = 0; g < kIssue / 4; ++g) mbar_init(&sm.gbar[g], 1);
        sm.gfail = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        if (!moe) {
            sm.exl[l0 & 1][0] = p.ex[size_t(l0) * p.E];
            sm.route_e[0] = sm.route_e[1] = 0;
            sm.route_w[0] = 1.f;
            sm.route_w[1] = 0.f;
        }
    }
    __syncwarp();
    // routed decode, warp 1: layer ln's router columns of this CTA into shared
    // memory as floats, in the upper half of the column-slice space (free from
    // the share until the next layer's biases; the lower half takes the
    // slice of r + y); every load is issued before any is stored
    constexpr int kRtsOff = kMaxSliceCols / 2;
    const bool rts_ok = moe && !predict && p.E * ncol <= kRtsOff && ncol <= kRtsOff;
    auto load_router_cols = [&](int ln) {
        const __half *R = reinterpret_cast<const __half *>(p.router[ln]);
        const int n = p.E * ncol;
        for (int i0 = 0; i0 < n; i0 += 32 * 8) {
            __half v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = i0 + 32 * u + lane;
                const int e = i / ncol, j = i - e * ncol;
                v[u] = i < n ? R[size_t(e) * d + c0 + j] : __float2half(0.f);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int i = i0 + 32 * u + lane;
                if (i < n) sm.rsl[kRtsOff + i] = __half2float(v[u]);
            }
        }
    };
    if (rts_ok && warp == 1) load_router_cols(l0);
    if (warp == 0 && vsm) stage_next_dense(l0);
    vpend = vsm;
    if (vsm && ns > 0) {
        staged_early = pending = true;
        upart2 = ufirst < u_round0;
    }
    cta_sync();

    // t value k of `ntr` (the layer's experts' ranks together) into shared memory
    uint16_t *const tpart = reinterpret_cast<uint16_t *>(sm.tsm);
    auto put_t = [&](int k, float tv, int ntr) {
        if constexpr (PF == kF32) sm.tsm[k] = tv;
        else if constexpr (PF == kI8) (void)tv;   // t goes in as digits, written after the poll
        else split_parts<PF>(tv, (PF == kBF16 && 3 * ntr <= 2 * kMaxRankTotal) ? 3 : 2, tpart + k, ntr);
    };

    // x of the current layer: this thread's vectors v = tid + kThreads k of
    // EPVW elements (the weight format's vector layout)
    float xw[MAXVW * EPVW];
    // EPVW elements of a predictor-format row from element e0 on, as floats
    static_assert(EPVW % EPVP == 0, "a weight vector spans whole predictor vectors");
    auto ld_pf = [&](const uint8_t *row, int e0, float *w) {
        constexpr int PB = PF == kF32 ? 4 : (PF == kI8 ? 1 : 2);
#pragma unroll
        for (int j = 0; j < EPVW / EPVP; ++j)
            cvt<PF>(*reinterpret_cast<const VP *>(row + size_t(e0 + j * EPVP) * PB), w + j * EPVP);
    };
    // rows [row0, row0 + n) of layer ln's experts' V (rows of t) at the
    // start of the staging buffer, in one round on stage_bar (thread 0)
    auto issue_vrows = [&](int ln, int row0, int n) {
        mbar_arrive_tx(&sm.stage_bar, uint32_t(n) * p.vrow);
        for (int rr = 0; rr < n;) {
            const int row = row0 + rr, e = row / r;
            const int cnt = min(n - rr, (e + 1) * r - row);
            stage_copy(stg + size_t(rr) * p.vrow, sm.exl[ln & 1][e].V + size_t(row - e * r) * p.vrow,
                       uint32_t(cnt) * p.vrow, &sm.stage_bar);
            rr += cnt;
        }
    };

    // -----------------------------------------------------------------------
    // Input of layer ln.  In the prologue (lp < l0) r is the caller's input;
    // otherwise it is the input of layer lp plus the fixed-point total of lp's
    // y, and every CTA forms all of it.  This CTA's columns are written out
    // (the next input buffer, the trace, or the caller's residual after the
    // last layer); x = RMSNorm(r) goes to xw (the predictor call takes x as
    // given); a routed layer picks its experts; this CTA's rows of t = V x go
    // out as tagged slots, which every CTA polls at the layer's start.  The
    // last layer stops after writing the residual, and a one-layer call that
    // emits y stops after writing y.  False if a bounded wait ran out.
    // -----------------------------------------------------------------------
    auto form_input = [&](int lp, int ln, long long *cycb) -> bool {
        const bool first = lp < l0;
        const bool emit = !first && p.y_out != nullptr;
        const bool last = ln >= l1;
        const int lip = lp - l0;   // profiling row (the layer whose tail this is)
        if (moe && !predict && !emit && !last && warp == 1 && lane < p.E)
            sm.exall[lane] = p.ex[size_t(ln) * p.E + lane];
        float rv[MAXVW * EPVW];
        {
            const float *rin = first ? (predict ? p.x_in : p.resid) : p.rbuf + size_t(lp & 1) * d;
            const unsigned long long *yt = first ? nullptr : p.yfix + size_t(lp & 1) * d;
            unsigned long long yq[MAXVW * EPVW];
            // every load first (one round trip), then the arithmetic
#pragma unroll
            for (int k = 0; k < MAXVW; ++k) {
                const int v = tid + kThreads * k;
#pragma unroll
                for (int i = 0; i < EPVW; i += 4) {
                    float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (v < nvecW && !emit) q = __ldcg(reinterpret_cast<const float4 *>(rin + v * EPVW + i));
                    rv[k * EPVW + i] = q.x; rv[k * EPVW + i + 1] = q.y;
                    rv[k * EPVW + i + 2] = q.z; rv[k * EPVW + i + 3] = q.w;
                }
                if (!first) {
#pragma unroll
                    for (int i = 0; i < EPVW; i += 2) {
                        ulonglong2 q = make_ulonglong2(0ull, 0ull);
                        if (v < nvecW) q = __ldcg(reinterpret_cast<const ulonglong2 *>(yt + v * EPVW + i));
                        yq[k * EPVW + i] = q.x;
                        yq[k * EPVW + i + 1] = q.y;
                    }
                }
            }
            if (!first) {
#pragma unroll
                for (int j = 0; j < MAXVW * EPVW; ++j)
                    rv[j] += float(double(static_cast<long long>(yq[j])) * (1.0 / 4294967296.0));
            }
        }
        if (lip >= 0) prof_put(p, lip, 20, gtimer());
        // this CTA's columns [c0, c0 + ncol)
        if (!predict) {
            float *dst = emit ? p.y_out : (last ? p.resid : p.rbuf + size_t(ln & 1) * d);
            float *trc = (!emit && !last && p.trace) ? p.trace + size_t(ln - l0) * d : nullptr;
            unsigned long long *yz = first ? p.yfix + size_t(l0 & 1) * d : nullptr;
#pragma unroll
            for (int k = 0; k < MAXVW; ++k) {
                const int v = tid + kThreads * k;
#pragma unroll
                for (int i = 0; i < EPVW; ++i) {
                    const int e = v * EPVW + i;
                    if (v < nvecW && e >= c0 && e < c0 + ncol) {
                        __stcg(dst + e, rv[k * EPVW + i]);
                        if (moe) sm.rsl[e - c0] = rv[k * EPVW + i];   // for the router's share
                        if (trc) __stcg(trc + e, rv[k * EPVW + i]);
                        if (yz) yz[e] = 0ull;   // layer l0's fixed-point total starts at zero
                    }
                }
            }
        }
        if (emit || last) return true;
        // x = RMSNorm(r): every CTA sums the same squares in the same order
        float inv = 1.f;
        if (!predict) {
            float ss = 0.f;
#pragma unroll
            for (int j = 0; j < MAXVW * EPVW; ++j) ss = fmaf(rv[j], rv[j], ss);
            ss = warp_sum(ss);
            if (lane == 0) sm.red[rb][warp][0] = ss;
            cta_sync();
            float tot = 0.f;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) tot += sm.red[rb][w][0];
            rb ^= 1;
            if (tid == 0 && !(tot <= 3.0e38f)) set_error(p.err, kDevCheck);   // sum of squares out of range
            inv = 1.f / sqrtf(tot / float(d) + p.eps);
        }
#pragma unroll
        for (int j = 0; j < MAXVW * EPVW; ++j) xw[j] = rv[j] * inv;
        if (lip >= 0) prof_put(p, lip, 7, gtimer());

        if constexpr (moe) {
            if (!predict) {
                // router logits W_r x: each CTA adds its columns' share in 64-bit
                // fixed point (integer adds: the totals do not depend on their
                // order); after a grid barrier every CTA reads the E totals and
                // takes the same decision: softmax over E, the two largest
                // (ties: lower index), renormalised
                unsigned long long *rl = reinterpret_cast<unsigned long long *>(p.bar + kRouterWord) +
                                         size_t(ln & 1) * kMaxExperts;
                if (warp < p.E && ncol > 0) {
                    // warp e: expert e's dot over this CTA's columns
                    const __half *R = reinterpret_cast<const __half *>(p.router[ln]);
                    const bool staged = rts_ok;   // this CTA's router columns already in shared memory
                    const int e = warp;
                    float q = 0.f;
                    for (int j = lane; j < ncol; j += 32) {
                        const float w = staged ? sm.rsl[kRtsOff + e * ncol + j] : __half2float(R[size_t(e) * d + c0 + j]);
                        q = fmaf(w, sm.rsl[j], q);
                    }
                    q = warp_sum(q);
                    if (lane == 0) red_add_u64(rl + e, fix_q(q * inv, p.err));
                }
                if (lip >= 0) prof_put(p, lip, 22, gtimer());
                grid_arrive(p, epoch);
                if (!grid_wait(&sm, p, epoch, bci, cycb)) return false;
                if (lip >= 0) prof_put(p, lip, 23, gtimer());
                if (warp == 0) {
                    // lane e holds expert e's logit.  The softmax is increasing
                    // in the logit, so the two largest probabilities are the two
                    // largest logits (ties: lower index), found by two warp
                    // argmax butterflies, and the renormalised pair
                    // p_a / (p_a + p_b) = 1 / (1 + exp(l_b - l_a)) needs one
                    // exponential, taken of a non-positive difference
                    const float lg = lane < p.E ? float(double(static_cast<long long>(__ldcg(rl + lane))) *
                                                        (1.0 / 4294967296.0))
                                                : -INFINITY;
                    auto argmax = [&](float v) -> int {
                        int i = lane;
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) {
                            const float vo = __shfl_xor_sync(0xffffffffu, v, o);
                            const int io = __shfl_xor_sync(0xffffffffu, i, o);
                            if (vo > v || (vo == v && io < i)) {
                                v = vo;
                                i = io;
                            }
                        }
                        return i;
                    };
                    const int ea = argmax(lg);
                    const int eb = argmax(lane == ea ? -INFINITY : lg);
                    const float la = __shfl_sync(0xffffffffu, lg, ea), lb = __shfl_sync(0xffffffffu, lg, eb);
                    if (lane == 0) {
                        const float q = expf(lb - la);   // p_b / p_a <= 1
                        const float wa = 1.f / (1.f + q), wb = q / (1.f + q);
                        const int lo = min(ea, eb), hi = max(ea, eb);
                        sm.route_e[0] = lo;
                        sm.route_e[1] = hi;
                        sm.route_w[0] = lo == ea ? wa : wb;
                        sm.route_w[1] = lo == ea ? wb : wa;
                        sm.exl[ln & 1][0] = sm.exall[lo];
                        sm.exl[ln & 1][1] = sm.exall[hi];
                        if (p.stats && b == 0) {
                            p.stats[(ln - l0) * 4 + 2] = lo;
                            p.stats[(ln - l0) * 4 + 3] = hi;
                        }
                    }
                }
            } else if (tid == 0) {
                // the predictor call: the caller's expert
                sm.route_e[0] = p.pred_expert;
                sm.route_w[0] = 1.f;
                sm.exl[ln & 1][0] = p.ex[size_t(ln) * p.E + p.pred_expert];
            }
            cta_sync();
            if (lip >= 0) prof_put(p, lip, 18, gtimer());
        }

        // this CTA's rows of t = V x: each thread dots its x elements with the
        // staged rows' same elements; one transposing warp reduction per round
        const int per = vsm ? nrows : min(kRA, kStageBytes / p.vrow);
        const int vb = vsm ? voff : 0;
        for (int row0 = a0; row0 < a1; row0 += per) {
            const int n = min(per, a1 - row0);
            if (vsm) {
                if (!stage_wait(&sm, p, vpar, bci, nullptr, &sm.vbar)) return false;
                vpend = false;
            } else {
                if (tid == 0) issue_vrows(ln, row0, n);
                pending = true;
                if (!stage_wait(&sm, p, spar, bci)) return false;
                pending = false;
            }
            if (row0 == a0 && lip >= 0) prof_put(p, lip, 19, gtimer());
            // routed: the experts' U strips (needed at the layer's start) start
            // moving towards L2 once the first V rows have landed, issued by a
            // thread that neither polls nor releases a grid barrier
            if (moe && row0 == a0 && tid == kThreads - 32 && ns > 0)
                for (int e = 0; e < ntop; ++e)
                    prefetch_l2(sm.exl[ln & 1][e].U + size_t(s0) * p.urow, uint32_t(ns) * p.urow);
            // four rows at a time, two groups of four in flight; after the
            // reduction lanes 8q .. 8q + 7 hold row g + q of the round
#pragma unroll 2
            for (int g = 0; g < n; g += 4) {
                float part[4];
#pragma unroll
                for (int rr = 0; rr < 4; ++rr) {
                    part[rr] = 0.f;
                    if (g + rr < n) {
                        const uint8_t *row = stg + vb + size_t(g + rr) * p.vrow;
#pragma unroll
                        for (int k = 0; k < MAXVW; ++k) {
                            const int v = tid + kThreads * k;
                            if (v < nvecW) {
                                float w[EPVW];
                                ld_pf(row, v * EPVW, w);
#pragma unroll
                                for (int i = 0; i < EPVW; ++i) part[rr] = fmaf(w[i], xw[k * EPVW + i], part[rr]);
                            }
                        }
                    }
                }
                const float s = warp_transpose_sum<4>(part);
                if ((lane & 7) == 0 && g + (lane >> 3) < n) sm.red[rb][warp][g + (lane >> 3)] = s;
            }
            cta_sync();
            if (tid < n) {
                float t = 0.f;
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) t += sm.red[rb][w][tid];
                if constexpr (PF == kI8) {
                    const int row = row0 + tid, e = row / r;
                    t *= __ldg(sm.exl[ln & 1][e].sV + (row - e * r));
                }
                st_relaxed_u64(tslot + row0 + tid, (static_cast<unsigned long long>(ln - l0 + 1) << 32) |
                                                       __float_as_uint(t));
            }
            rb ^= 1;
        }
        if (lip >= 0) prof_put(p, lip, 5, gtimer());
        // The rows of t travel as tagged slots, which every CTA polls at the
        // layer's start: no grid barrier.  The prologue alone keeps one, so
        // that every CTA's zeroing of layer l0's fixed-point total is ordered
        // before any CTA's reduction into it.  The first U round of layer ln
        // (or the piece of it that waited for the V rows' space) lands during
        // the wait; issued after the arrival, whose release would otherwise
        // wait for the copies.
        const bool pbar = first && !predict;
        if (pbar) grid_arrive(p, epoch);
        if (ns > 0 && warp == 0) {
            if (vsm) {
                if (upart2) stage_u_at(sm.exl[ln & 1][0], ufirst, u_round0 - ufirst, ufirst, true);
            } else if (both_u) {
                stage_u_at(sm.exl[ln & 1][0], 0, ns, 0, false);
                stage_u_at(sm.exl[ln & 1][1], 0, ns, u2, true);
            } else {
                stage_u(sm.exl[ln & 1][0], 0, min(ns, ucap));
                if (!moe && lane == 0 && ns > ucap)
                    prefetch_l2(sm.exl[ln & 1][0].U + size_t(s0 + ucap) * p.urow, uint32_t(ns - ucap) * p.urow);
            }
        }
        if (vsm) upart2 = false;
        else if (ns > 0) staged_early = pending = true;
        return pbar ? grid_wait(&sm, p, epoch, bci, cycb) : true;
    };

    // INT4 weights: x's digits in the gather dots' B layout, for k-group G
    // (32 elements), column p (digit p; columns 5..7 zero) and lane quad tq, 8
    // bytes: digit p of elements 8 tq + 0, 2, 4, 6, then of 8 tq + 1, 3, 5, 7
    // (the order of i4x8_to_s8).  The thread holding vector v = 4 G + tq
    // writes them, while the CTA waits at the balance step.
    auto write_digits = [&]() {
        if constexpr (WF == kI4) {
#pragma unroll
            for (int k = 0; k < MAXVW; ++k) {
                const int v = tid + kThreads * k;
                if (v < nvecW) {
                    uint32_t dg[5][2] = {};
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        float t = xw[k * EPVW + i] * xs;
#pragma unroll
                        for (int q = 0; q < 5; ++q) {
                            const float r = rintf(t);
                            dg[q][i & 1] |= (uint32_t(int(r)) & 0xffu) << (8 * (i >> 1));
                            t = (t - r) * 128.f;
                        }
                    }
                    uint2 *dst = reinterpret_cast<uint2 *>(stg + xpoff) + size_t(v >> 2) * 32 + (v & 3);
#pragma unroll
                    for (int q = 0; q < 5; ++q) dst[q * 4] = make_uint2(dg[q][0], dg[q][1]);
#pragma unroll
                    for (int q = 5; q < 8; ++q) dst[q * 4] = make_uint2(0u, 0u);
                }
            }
        }
    };

    // Each pass forms the input of layer l + 1 and then runs that layer; the
    // first pass (l = l0 - 1) is the prologue.  One call site keeps one copy
    // of the input step's code.
    long long cyc_a = 0, cyc_b = 0, cyc_c = 0, cyc_bar = 0;
    for (int l = l0 - 1;;) {
        // ---------------- the next layer's input, routing and t --------------
        if (!form_input(l, l + 1, &cyc_bar)) break;
        if (l >= l0) {
            prof_put(p, l - l0, 6, gtimer());
            prof_put(p, l - l0, 10, cyc_a);
            prof_put(p, l - l0, 11, cyc_b);
            prof_put(p, l - l0, 12, cyc_c);
            prof_put(p, l - l0, 13, cyc_bar);
        }
        if (++l >= l1) break;
        const int li = l - l0;
        cyc_a = cyc_b = cyc_c = cyc_bar = 0;
        prof_put(p, li, 0, gtimer());
        const long long ca0 = clock64();

        // ---------------- the layer's t and biases ---------------------------
        for (int e = 0; e < ntop; ++e)
            for (int i = tid; i < ns; i += kThreads) sm.cbuf[e][i] = __ldg(sm.exl[l & 1][e].c + s0 + i);
        // the next layer's weight pointers (dense), for its prefetches during this layer
        if (!moe && tid == kThreads - 1 && l + 1 < l1) sm.exl[(l + 1) & 1][0] = p.ex[size_t(l + 1) * p.E];
        // layer l - 1's fixed-point total (read before the last merge barrier)
        // is cleared for layer l + 1
        if (!predict && l + 1 < l1) {
            unsigned long long *yz = p.yfix + size_t((l + 1) & 1) * d;
            for (int e = c0 + tid; e < c0 + ncol; e += kThreads) yz[e] = 0ull;
        }
        // routed: layer l - 1's router totals (read before the last merge
        // barrier) are cleared for layer l + 1
        if (moe && !predict && b == 0 && tid < kMaxExperts && l + 1 < l1)
            reinterpret_cast<unsigned long long *>(p.bar + kRouterWord)[size_t((l + 1) & 1) * kMaxExperts + tid] = 0ull;
        if (!moe && tid == 0 && p.stats && b == 0 && !predict) {
            p.stats[li * 4 + 2] = -1;
            p.stats[li * 4 + 3] = -1;
        }
        // the rows of t: each thread polls its slots until all of them carry
        // this layer's tag (bounded by wait_ns), then keeps the values
        bool tok = true;
        {
            constexpr int kTS = kMaxRankTotal / kThreads;
            static_assert(kTS * kThreads == kMaxRankTotal && kTS <= 32, "whole slots per thread");
            const int nt = ntop * r;
            // (PI_DEBUG_STALL_T_POLL: a tag that no layer writes)
            const unsigned tg = unsigned(l - l0 + 1) + ((p.debug_flags & 8) ? 0x40000000u : 0u);
            unsigned long long w[kTS];
            unsigned need = 0;
#pragma unroll
            for (int i = 0; i < kTS; ++i) {
                const int k = tid + i * kThreads;
                w[i] = k < nt ? ld_relaxed_u64(tslot + k) : 0ull;
                if (k < nt && unsigned(w[i] >> 32) != tg) need |= 1u << i;
            }
            if (need) {
                const long long t0 = gtimer();
                for (unsigned it = 1;; ++it) {
#pragma unroll
                    for (int i = 0; i < kTS; ++i)
                        if ((need >> i) & 1u) {
                            w[i] = ld_relaxed_u64(tslot + tid + i * kThreads);
                            if (unsigned(w[i] >> 32) == tg) need &= ~(1u << i);
                        }
                    if (!need) break;
                    if ((it & 31) == 0 && gtimer() - t0 > p.wait_ns) {
                        set_error(p.err, kDevTimeout);
                        tok = false;
                        break;
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < kTS; ++i) {
                const int k = tid + i * kThreads;
                if (k < nt) put_t(k, __uint_as_float(unsigned(w[i])), nt);
            }
            if constexpr (PF == kI8) {
                // 8-bit predictor: each warp's bound of |t|, gathered through
                // the block barrier below
                float mx = 0.f;
#pragma unroll
                for (int i = 0; i < kTS; ++i)
                    if (tid + i * kThreads < nt) mx = fmaxf(mx, fabsf(__uint_as_float(unsigned(w[i]))));
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                if (lane == 0) sm.red[rb][warp][0] = mx;
            }
            if (!__syncthreads_and(tok)) break;
            if constexpr (PF == kI8) {
                // t as signed base-128 digits for the integer logits.  The
                // bound of |t| over the layer (the same in every CTA) gives
                // ts = 2^(6 - e), max |t| < 2^e, so t * ts lies in (-64, 64);
                // digit 0 is its nearest integer and each further digit the
                // nearest integer of 128 times the remainder (every step exact;
                // four digits leave below 2^-22 2^(e-6)).  Adding 1.5 * 2^23
                // rounds to the nearest integer and leaves it, two's
                // complement, in the low byte of the sum's bits.
                float mx = 0.f;
#pragma unroll
                for (int w2 = 0; w2 < kConsumerWarps; ++w2) mx = fmaxf(mx, sm.red[rb][w2][0]);
                rb ^= 1;
                int ex = 0;
                (void)frexpf(mx, &ex);
                tsc = ldexpf(1.f, 6 - ex);
                // the digits of four consecutive t values form one 32-bit word
                // (byte j = element 4q + j): for expert slot e, k32 step s,
                // digit p and lane quad tq, the word pair of elements 32 s +
                // 4 tq .. + 3 and 32 s + 16 + 4 tq .. + 3 (the B fragment)
                uint32_t *dw = reinterpret_cast<uint32_t *>(sm.tsm);
                const int nk32 = r >> 5;
#pragma unroll
                for (int i = 0; i < kTS; ++i) {
                    const int k = tid + i * kThreads;
                    if (k < nt) {   // the same in every lane of a warp (nt is a multiple of 32)
                        float v = __uint_as_float(unsigned(w[i])) * tsc;
                        uint32_t db[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float m = v + 12582912.f;
                            db[q] = (__float_as_uint(m) & 0xffu) << (8 * (lane & 3));
                            v = (v - (m - 12582912.f)) * 128.f;
                        }
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            db[q] |= __shfl_xor_sync(0xffffffffu, db[q], 1);
                            db[q] |= __shfl_xor_sync(0xffffffffu, db[q], 2);
                        }
                        if ((lane & 3) == 0) {
                            const int e = k / r, kk = k - e * r, st = kk >> 5, qd = (kk & 31) >> 2;
#pragma unroll
                            for (int q = 0; q < 4; ++q)
                                dw[(((e * nk32 + st) * 4 + q) * 4 + (qd & 3)) * 2 + (qd >> 2)] = db[q];
                        }
                    }
                }
            }
        }

        cyc_a = clock64() - ca0;
        prof_put(p, li, 1, gtimer());

        // ---------------- z = U t - c over the strip, compaction -------------
        const long long cb0 = clock64();
        {
            bool ok = true;
            for (int e = 0; e < ntop && ok; ++e) {
                // fp32 predictor: this lane's t values (the columns of its U vectors)
                float tu[PF == kF32 ? kMaxU * EPVP : 1];
                if constexpr (PF == kF32) {
#pragma unroll
                    for (int k = 0; k < kMaxU; ++k) {
                        const int v = lane + 32 * k;
#pragma unroll
                        for (int i = 0; i < EPVP; i += 4) {
                            float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
                            if (v < nvecU) q = *reinterpret_cast<const float4 *>(sm.tsm + e * r + v * EPVP + i);
                            tu[k * EPVP + i] = q.x; tu[k * EPVP + i + 1] = q.y;
                            tu[k * EPVP + i + 2] = q.z; tu[k * EPVP + i + 3] = q.w;
                        }
                    }
                }
                for (int row0 = 0; row0 < ns && ok; row0 += ucap) {
                    const int n = min(ucap, ns - row0);
                    // the second expert's strip landed with the first's
                    const bool second = both_u && e == 1;
                    const uint8_t *ust = stg + (second ? size_t(u2) * p.urow : 0);
                    if (!second) {
                        if (!(staged_early && row0 == 0)) {
                            if (warp == 0) stage_u(sm.exl[l & 1][e], row0, n);
                        }
                        staged_early = false;
                        pending = true;
                        if (!stage_wait(&sm, p, spar, bci, &cyc_b)) { ok = false; break; }
                        pending = false;
                    }
                    if (e == 0 && row0 == 0) prof_put(p, li, 14, gtimer());
                    if constexpr (PF == kF32) {
                        // each warp takes rows warp, warp + 16, ...; four rows at a time,
                        // each with its own accumulators, to keep the dependent FMA and
                        // shuffle chains of different rows overlapped
                        constexpr int kZR = 4;
                        for (int rr0 = warp; rr0 < n; rr0 += kConsumerWarps * kZR) {
                            float a[kZR][2];
    #pragma unroll
                            for (int j = 0; j < kZR; ++j) {
                                a[j][0] = 0.f;
                                a[j][1] = 0.f;
                                const int rr = rr0 + j * kConsumerWarps;
                                if (rr < n) {
                                    const uint8_t *urow = ust + size_t(rr) * p.urow;
    #pragma unroll
                                    for (int k = 0; k < kMaxU; ++k) {
                                        const int v = lane + 32 * k;
                                        if (v < nvecU) {
                                            float w[EPVP];
                                            cvt<PF>(*reinterpret_cast<const VP *>(urow + v * VBP), w);
    #pragma unroll
                                            for (int i = 0; i < EPVP; ++i)
                                                a[j][i & 1] = fmaf(w[i], tu[k * EPVP + i], a[j][i & 1]);
                                        }
                                    }
                                }
                            }
    #pragma unroll
                            for (int j = 0; j < kZR; ++j) a[j][0] += a[j][1];
    #pragma unroll
                            for (int o = 16; o > 0; o >>= 1)
    #pragma unroll
                                for (int j = 0; j < kZR; ++j) a[j][0] += __shfl_xor_sync(0xffffffffu, a[j][0], o);
                            if (lane == 0) {
    #pragma unroll
                                for (int j = 0; j < kZR; ++j) {
                                    const int rr = rr0 + j * kConsumerWarps;
                                    if (rr < n) {
                                        const int loc = row0 + rr;
                                        const float z = a[j][0] - sm.cbuf[e][loc];
                                        sm.zbuf[e][loc] = z;
                                        if (predict && p.z_out) p.z_out[s0 + loc] = z;
                                    }
                                }
                            }
                        }
                    } else if constexpr (PF == kI8) {
                        // integer tensor-core dots of signed-byte U rows: A = 16
                        // staged rows x 32 bytes (ldmatrix; rows stored
                        // chunk-permuted by row mod 8 when u_swz, as the 16-bit
                        // rows), B = t's digits (column p = digit p), D exact in
                        // int32 over the warp's k32 steps; warp w takes steps
                        // w, w + 16, ...
                        const int nks = r >> 5, nmt = (n + 15) / 16;
                        const int g = lane >> 2, tq = lane & 3;
                        const int arow = lane & 15;
                        const uint2 *bd = reinterpret_cast<const uint2 *>(sm.tsm) + size_t(e) * nks * 16 + tq;
                        // this lane's digit columns 2 tq and 2 tq + 1: weights 2^-7p / ts
                        const float dw0 = tq < 2 ? ldexpf(1.f, -14 * tq) / tsc : 0.f;
                        const float dw1 = tq < 2 ? ldexpf(1.f, -14 * tq - 7) / tsc : 0.f;
                        // m-tiles per pass: seven keep a 97-row strip (F = 14336 over 148
                        // CTAs) in one pass; the fp16-weight kernels keep five (74-row
                        // strips, F = 11008)
                        constexpr int kZT = MAXVW > 1 ? 4 : (WF == kF16 ? 5 : 7);
                        for (int mt0 = 0; mt0 < nmt; mt0 += kZT) {
                            int c[kZT][4];
#pragma unroll
                            for (int t = 0; t < kZT; ++t) c[t][0] = c[t][1] = c[t][2] = c[t][3] = 0;
                            int arw[kZT];
#pragma unroll
                            for (int t = 0; t < kZT; ++t) arw[t] = min((mt0 + t) * 16 + arow, n - 1);
                            const uint32_t sbase = s2u(ust);
                            for (int ks = warp; ks < nks; ks += kConsumerWarps) {
                                uint2 bx = make_uint2(0u, 0u);
                                if (g < 4) bx = bd[(ks * 4 + g) * 4];
                                const int chunk = 2 * ks + (lane >> 4);   // 16-byte chunk of the row
#pragma unroll
                                for (int t0 = 0; t0 < kZT; t0 += 3) {
                                    uint32_t a[3][4];
#pragma unroll
                                    for (int t = t0; t < t0 + 3; ++t) {
                                        if (t < kZT && mt0 + t < nmt) {
                                            const int key = p.u_swz ? (arw[t] & 7) : 0;
                                            ldsm_x4_a(sbase + uint32_t(arw[t]) * uint32_t(p.urow) +
                                                          uint32_t(((chunk & ~7) | ((chunk ^ key) & 7)) << 4),
                                                      a[t - t0]);
                                        }
                                    }
#pragma unroll
                                    for (int t = t0; t < t0 + 3; ++t)
                                        if (t < kZT && mt0 + t < nmt)
                                            imma16832_acc(c[t], a[t - t0][0], a[t - t0][1], a[t - t0][2], a[t - t0][3],
                                                          bx.x, bx.y);
                                }
                            }
                            // the digit columns sit in the four lanes of a quad
#pragma unroll
                            for (int t = 0; t < kZT; ++t) {
                                float z0 = fmaf(float(c[t][0]), dw0, float(c[t][1]) * dw1);
                                float z1 = fmaf(float(c[t][2]), dw0, float(c[t][3]) * dw1);
                                z0 += __shfl_xor_sync(0xffffffffu, z0, 1);
                                z1 += __shfl_xor_sync(0xffffffffu, z1, 1);
                                z0 += __shfl_xor_sync(0xffffffffu, z0, 2);
                                z1 += __shfl_xor_sync(0xffffffffu, z1, 2);
                                if (tq == 0 && mt0 + t < nmt) {
                                    sm.zred[warp][(mt0 + t) * 16 + g] = z0;
                                    sm.zred[warp][(mt0 + t) * 16 + g + 8] = z1;
                                }
                            }
                        }
                        cta_sync();
                        const int nw = min(kConsumerWarps, nks);
                        const float *su = sm.exl[l & 1][e].sU + s0 + row0;
                        for (int rr = tid; rr < n; rr += kThreads) {
                            float q[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                            for (int w = 0; w < kConsumerWarps; ++w)
                                if (w < nw) q[w & 3] += sm.zred[w][rr];
                            const float a = (q[0] + q[1]) + (q[2] + q[3]);
                            const int loc = row0 + rr;
                            const float z = a * __ldg(su + rr) - sm.cbuf[e][loc];
                            sm.zbuf[e][loc] = z;
                            if (predict && p.z_out) p.z_out[s0 + loc] = z;
                        }
                    } else {
                        // tensor-core dots: A = 16 staged U rows x 16 columns
                        // (ldmatrix; rows stored chunk-permuted by row mod 8
                        // when u_swz), B = the matching 16 entries of t as
                        // 16-bit parts (part g in column g), fp32
                        // accumulators; warp w takes k-steps w, w + 16, ...
                        constexpr int kParts = PF == kBF16 ? 3 : 2;
                        const int ntr = ntop * r;
                        const int nparts = (PF == kBF16 && 3 * ntr <= 2 * kMaxRankTotal) ? 3 : 2;
                        const int nks = r / 16, nmt = (n + 15) / 16;
                        const int g = lane >> 2, tq = lane & 3;
                        const int arow = lane & 15;                       // row within an m-tile
                        const uint16_t *bpart = tpart + g * ntr + e * r + 2 * tq;
                        // m-tiles in passes of kZT (bounded accumulator registers)
                        // m-tiles per pass: seven keep a 97-row strip (F = 14336 over 148
                        // CTAs) in one pass; the fp16-weight kernels keep five, exactly
                        // their 74-row strips (F = 11008): accumulators for tiles a strip
                        // does not have cost registers (measured: 0.5-0.8% per layer
                        // against eight and six)
                        constexpr int kZT = MAXVW > 1 ? 4 : (WF == kF16 ? 5 : 7);
                        for (int mt0 = 0; mt0 < nmt; mt0 += kZT) {
                            float c[kZT][4];
#pragma unroll
                            for (int t = 0; t < kZT; ++t) c[t][0] = c[t][1] = c[t][2] = c[t][3] = 0.f;
                            // this lane's row in each m-tile (rows past the round's last are
                            // read as its last row; their results are never used); its chunk
                            // permutation key is the staged row mod 8 (rounds start at
                            // multiples of 8)
                            int arw[kZT];
#pragma unroll
                            for (int t = 0; t < kZT; ++t) arw[t] = min((mt0 + t) * 16 + arow, n - 1);
                            const uint32_t sbase = s2u(ust);
                            for (int ks = warp; ks < nks; ks += kConsumerWarps) {
                                uint32_t b0 = 0u, b1 = 0u;
                                if (g < nparts) {
                                    b0 = *reinterpret_cast<const uint32_t *>(bpart + ks * 16);
                                    b1 = *reinterpret_cast<const uint32_t *>(bpart + ks * 16 + 8);
                                }
                                const int chunk = 2 * ks + (lane >> 4);            // 16-byte chunk of the row
                                // the matrix loads of three m-tiles first, then their MMAs,
                                // so that the loads' latencies overlap
#pragma unroll
                                for (int t0 = 0; t0 < kZT; t0 += 3) {
                                    uint32_t a[3][4];
#pragma unroll
                                    for (int t = t0; t < t0 + 3; ++t) {
                                        if (t < kZT && mt0 + t < nmt) {
                                            const int key = p.u_swz ? (arw[t] & 7) : 0;
                                            ldsm_x4_a(sbase + uint32_t(arw[t]) * uint32_t(p.urow) +
                                                          uint32_t(((chunk & ~7) | ((chunk ^ key) & 7)) << 4),
                                                      a[t - t0]);
                                        }
                                    }
#pragma unroll
                                    for (int t = t0; t < t0 + 3; ++t)
                                        if (t < kZT && mt0 + t < nmt)
                                            mma16816<PF>(c[t], a[t - t0][0], a[t - t0][1], a[t - t0][2], a[t - t0][3], b0, b1);
                                }
                            }
                            // sum over the parts: columns 0 and 1 sit in lane 4g, column 2 in lane 4g + 1
#pragma unroll
                            for (int t = 0; t < kZT; ++t) {
                                float z0 = c[t][0] + c[t][1], z1 = c[t][2] + c[t][3];
                                if constexpr (kParts == 3) {
                                    z0 += __shfl_down_sync(0xffffffffu, c[t][0], 1);
                                    z1 += __shfl_down_sync(0xffffffffu, c[t][2], 1);
                                }
                                if (tq == 0 && mt0 + t < nmt) {
                                    sm.zred[warp][(mt0 + t) * 16 + g] = z0;
                                    sm.zred[warp][(mt0 + t) * 16 + g + 8] = z1;
                                }
                            }
                        }
                        cta_sync();
                        if (e == 0 && row0 == 0) prof_put(p, li, 15, gtimer());
                        // across warps in fixed order: four interleaved partial sums
                        // (warps w, w + 4, ...), then those four in order
                        const int nw = min(kConsumerWarps, nks);
                        for (int rr = tid; rr < n; rr += kThreads) {
                            float q[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                            for (int w = 0; w < kConsumerWarps; ++w)
                                if (w < nw) q[w & 3] += sm.zred[w][rr];
                            const float a = (q[0] + q[1]) + (q[2] + q[3]);
                            const int loc = row0 + rr;
                            const float z = a - sm.cbuf[e][loc];
                            sm.zbuf[e][loc] = z;
                            if (predict && p.z_out) p.z_out[s0 + loc] = z;
                        }
                    }
                    cta_sync();   // the staging buffer is reused by the next round
                }
            }
            if (!ok) break;
        }
        prof_put(p, li, 9, gtimer());
        // compaction in ascending strip order: warp e builds expert slot e's list
        if (warp < ntop) {
            const int e = warp;
            int cnt = 0;
            const int off = e == 0 ? 0 : kMaxStrip;
            for (int base = 0; base < ns; base += 32) {
                const int loc = base + lane;
                const bool act = loc < ns && sm.zbuf[e][loc] > p.threshold;
                const unsigned msk = __ballot_sync(0xffffffffu, act);
                if (act) {
                    const int pos = cnt + __popc(msk & ((1u << lane) - 1u));
                    sm.lst[off + pos] = int16_t((e << 12) | loc);
                    if (predict) p.lists[size_t(b) * kMaxStrip + pos] = s0 + loc;
                    if (p.masks) {
                        const int gp = s0 + loc;
                        const int words = (p.F + 31) / 32;
                        atomicOr(p.masks + (size_t(li) * ntop + e) * words + (gp >> 5), 1u << (gp & 31));
                    }
                }
                cnt += __popc(msk);
            }
            if (lane == 0) {
                sm.lst_n[e] = cnt;
                if (predict) p.counts[b] = cnt;
                if (p.stats && !predict) atomicAdd(p.stats + li * 4 + 0, cnt);
            }
        }
        cta_sync();
        (void)cb0;
        prof_put(p, li, 2, gtimer());

        if (predict) {
            // global ascending list: prefix of the strip counts, then copy
            if (!grid_sync(&sm, p, epoch, bci, &cyc_bar)) break;
            int pre = 0;
            for (int i = tid; i < b; i += kThreads) pre += __ldcg(p.counts + i);
            pre = __reduce_add_sync(0xffffffffu, pre);
            if (lane == 0) sm.red[rb][warp][0] = __int_as_float(pre);
            cta_sync();
            int base = 0;
            for (int w = 0; w < kConsumerWarps; ++w) base += __float_as_int(sm.red[rb][w][0]);
            const int cnt = sm.lst_n[0];
            for (int i = tid; i < cnt; i += kThreads) p.idx_out[base + i] = s0 + (sm.lst[i] & 0xfff);
            if (b == S - 1 && tid == 0) p.count_out[0] = base + cnt;
            break;
        }

        // ---------------- balance: equal shares of the active list -----------
        // Each strip publishes its active neurons (with their biases), arrives
        // at a grid barrier and starts their rows moving towards L2; after the
        // barrier every CTA takes an equal share [lo, hi) of the lists
        // concatenated in strip order.  The share depends only on the active
        // set, so the per-CTA partials and their fixed-order reduction stay
        // deterministic.
        const ExpertDev *exs[kMaxTopK] = {&sm.exl[l & 1][0], &sm.exl[l & 1][ntop > 1 ? 1 : 0]};
        if (p.local_gather) {
            // each CTA gathers its own strip's active neurons (the snake-dealt
            // table balances their expected number): no exchange, no barrier;
            // records past the first round start moving towards L2 at once
            const int n0 = sm.lst_n[0], nl = n0 + (ntop > 1 ? sm.lst_n[1] : 0);
            const int cap1 = min(kRound, kStageBytes / (kSpec ? p.rec_bytes : p.gu_bytes));
            for (int j = tid; j < nl; j += kThreads) {
                const int en = j < n0 ? sm.lst[j] : sm.lst[kMaxStrip + (j - n0)];
                const int e = en >> 12, loc = en & 0xfff, pos = s0 + loc;
                const unsigned code = rec_code(p.hot_k, b, loc, pos);
                sm.glst[j] = int(unsigned(e << 24) | code);
                sm.gc[j] = sm.cbuf[e][loc];
                if (j >= cap1 && !(code & kColdBit))
                    prefetch_l2(exs[e]->Wgu + size_t(code) * p.rec_bytes, uint32_t(kSpec ? p.rec_bytes : p.gu_bytes));
            }
            if (tid == 0) sm.share_n = nl;
            write_digits();
            cta_sync();
        } else {
        {
            const int n0 = sm.lst_n[0], nl = n0 + (ntop > 1 ? sm.lst_n[1] : 0);
            unsigned long long *pb = p.pub + size_t(b) * (kMaxTopK * kMaxStrip);
            for (int j = tid; j < nl; j += kThreads) {
                const int en = j < n0 ? sm.lst[j] : sm.lst[kMaxStrip + (j - n0)];
                const int e = en >> 12, loc = en & 0xfff, pos = s0 + loc;
                __stcg(pb + j, (unsigned long long)(unsigned(e << 24) | rec_code(p.hot_k, b, loc, pos)) |
                                   ((unsigned long long)__float_as_uint(sm.cbuf[e][loc]) << 32));
            }
            if (tid == 0) __stcg(p.counts + b, nl);
            // the rows start moving towards L2 once this CTA has arrived, so
            // that the arrival's release does not wait for them
            grid_arrive(p, epoch);
            for (int j = tid; j < nl; j += kThreads) {
                const int en = j < n0 ? sm.lst[j] : sm.lst[kMaxStrip + (j - n0)];
                const int e = en >> 12, loc = en & 0xfff;
                const unsigned code = rec_code(p.hot_k, b, loc, s0 + loc);
                if (!(code & kColdBit))
                    prefetch_l2(exs[e]->Wgu + size_t(code) * p.rec_bytes, uint32_t(kSpec ? p.rec_bytes : p.gu_bytes));
            }
            write_digits();
        }
        if (!grid_wait(&sm, p, epoch, bci, &cyc_bar)) break;
        prof_put(p, li, 16, gtimer());
        {
            // exclusive prefix of the strip counts (S <= 256: warps 0..7)
            const int cnt = tid < S ? __ldcg(p.counts + tid) : 0;
            int inc = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += v;
            }
            if (lane == 31) sm.red[rb][warp][0] = __int_as_float(inc);
            cta_sync();
            if (tid <= S) {
                int pre = inc - cnt;
                for (int w = 0; w < warp; ++w) pre += __float_as_int(sm.red[rb][w][0]);
                sm.scan[tid] = pre;
            }
            rb ^= 1;
            cta_sync();
            const int ntot = sm.scan[S];
            const int lo = int((long long)b * ntot / S), hi = int((long long)(b + 1) * ntot / S);
            for (int j = lo + tid; j < hi; j += kThreads) {
                int q0 = 0, q1 = S;   // strip q with scan[q] <= j < scan[q + 1]
                while (q1 - q0 > 1) {
                    const int mid = (q0 + q1) >> 1;
                    if (sm.scan[mid] <= j) q0 = mid;
                    else q1 = mid;
                }
                const unsigned long long w = __ldcg(p.pub + size_t(q0) * (kMaxTopK * kMaxStrip) + (j - sm.scan[q0]));
                sm.glst[j - lo] = int(unsigned(w));
                sm.gc[j - lo] = __uint_as_float(unsigned(w >> 32));
            }
            if (tid == 0) sm.share_n = hi - lo;
            cta_sync();
        }
        }

        // routed: the next layer's router columns land during the gather
        if (rts_ok && warp == 1 && l + 1 < l1) load_router_cols(l + 1);
        // ---------------- gather rows of active neurons ----------------------
        // Rounds of up to kRound neurons: one bulk-copy round brings their
        // W_gate/W_up records (and, when speculative, their W_down rows) into
        // shared memory; the dots of all of them are reduced at once.
        prof_put(p, li, 8, gtimer());
        const long long cc0 = clock64();
        const int m = sm.share_n;
        const int per_n = kSpec ? p.rec_bytes : p.gu_bytes;   // bytes per neuron in a round (its record)
        // records are issued in batches of up to kIssue (as many as the
        // staging buffer holds) and consumed in rounds of up to kRound, so a
        // round's dots overlap the later rounds' copies
        // slots of a batch, sstr bytes apart: INT4 records get 16 bytes of
        // padding, so that the tensor-core dots' eight rows per load fall in
        // different shared-memory banks
        const int sstr = WF == kI4 ? per_n + 16 : per_n;
        const int cap_all = min(kIssue, (WF == kI4 ? xpoff : kStageBytes) / sstr);
        const int cap_n = min(kRound, cap_all);
        int jb = 0, je = 0;   // the batch in shared memory: neurons [jb, je) in slots 0 ..

        // the next layer's V rows of this CTA and biases (dense) or router
        // rows (routed) start moving towards L2 now
        if (tid == kThreads - 1 && l + 1 < l1) {
            if (!moe) {
                if (nrows > 0) prefetch_l2(sm.exl[(l + 1) & 1][0].V + size_t(a0) * p.vrow, uint32_t(nrows) * p.vrow);
                if (ns > 0) {
                    const int c_lo = s0 & ~3, c_hi = (s0 + ns + 3) & ~3;   // 16-byte aligned, padded
                    prefetch_l2(sm.exl[(l + 1) & 1][0].c + c_lo, uint32_t(c_hi - c_lo) * 4);
                }
            } else if (ncol > 0) {
                // this CTA's columns of each router row (its share of the logits)
                for (int e = 0; e < p.E; ++e)
                    prefetch_l2(p.router[l + 1] + (size_t(e) * d + c0) * 2, uint32_t(ncol) * 2);
            }
        }

        float acc[MAXVW * EPVW];
#pragma unroll
        for (int i = 0; i < MAXVW * EPVW; ++i) acc[i] = 0.f;
        // acc += h * (a W_down row in shared memory)
        auto axpy_smem = [&](const uint8_t *row, float h) {
#pragma unroll
            for (int k = 0; k < MAXVW; ++k) {
                const int v = tid + kThreads * k;
                if (v < nvecW) {
                    float w[EPVW];
                    cvt<WF>(*reinterpret_cast<const VW *>(row + v * VBW), w);
                    float hs = h;
                    if constexpr (WF == kI4) hs = h * __half2float(*reinterpret_cast<const __half *>(row + d / 2 + (v >> 2) * 2));
#pragma unroll
                    for (int i = 0; i < EPVW; ++i) acc[k * EPVW + i] = fmaf(hs, w[i], acc[k * EPVW + i]);
                }
            }
        };
        // dot of a row in shared memory with this thread's x columns
        auto dot_smem = [&](const uint8_t *row) -> float {
            float a = 0.f;
#pragma unroll
            for (int k = 0; k < MAXVW; ++k) {
                const int v = tid + kThreads * k;
                if (v < nvecW) {
                    float w[EPVW];
                    cvt<WF>(*reinterpret_cast<const VW *>(row + v * VBW), w);
                    float c = 0.f;
#pragma unroll
                    for (int i = 0; i < EPVW; ++i) c = fmaf(w[i], xw[k * EPVW + i], c);
                    if constexpr (WF == kI4) c *= __half2float(*reinterpret_cast<const __half *>(row + d / 2 + (v >> 2) * 2));
                    a += c;
                }
            }
            return a;
        };

        bool gok = true;
        int nz_total = 0;            // neurons with h != 0 so far (list order)
        for (int j0 = 0, k = 0; j0 < m && gok; j0 += k) {
            if (j0 == je) {
                // the next batch: neurons [j0, je) into slots 0 .. je - j0 - 1
                jb = j0;
                je = min(m, j0 + cap_all);
                const int kb = je - jb;
                const int ngb = (kb + 3) / 4;   // groups of four neurons, one barrier each
                if (warp == 0) {
                    // lane 0 announces each group's bytes (records in HBM only), then
                    // lane n copies neuron n onto its group's barrier
                    const int en_l = lane < kb ? sm.glst[jb + lane] : 0;
                    const bool hot_l = lane < kb && !(unsigned(en_l) & kColdBit);
                    const unsigned hot_m = __ballot_sync(0xffffffffu, hot_l);
                    if (lane < ngb)
                        mbar_arrive_tx(&sm.gbar[lane], uint32_t(__popc((hot_m >> (4 * lane)) & 0xfu)) * per_n);
                    __syncwarp();
                    if (hot_l) {
                        const int e = en_l >> 24;
                        const unsigned code = unsigned(en_l) & 0xffffffu;
                        uint8_t *slot = stg + size_t(lane) * sstr;
                        uint64_t *gb = &sm.gbar[lane >> 2];
                        stage_copy(slot, exs[e]->Wgu + size_t(code) * p.rec_bytes, uint32_t(per_n), gb);
                    }
                }
                if (p.hot_k) {
                    // records in host memory: every thread copies pieces of them
                    for (int n = 0; n < kb; ++n) {
                        const int en = sm.glst[jb + n];
                        if (!(unsigned(en) & kColdBit)) continue;
                        const unsigned idx = unsigned(en) & (kColdBit - 1u);
                        copy_host_rec(stg + size_t(n) * sstr, exs[en >> 24]->Wgu_cold + size_t(idx) * p.rec_bytes,
                                      per_n, tid, kThreads);
                    }
                    cta_sync();
                }
                gpend = (1u << ngb) - 1u;
            }
            k = min(cap_n, je - j0);
            const int sb = j0 - jb;                                         // this round's first slot
            const unsigned rmask = ((1u << ((k + 3) / 4)) - 1u) << (sb >> 2);   // its groups
            // Dots of the round's neurons: values 2n (gate) and 2n + 1 (up),
            // each warp's partial over its own x vectors to sm.red.
            //
            // INT4 weights: integer tensor-core dots, one m-tile of 16 rows at
            // a time (gated: the gate rows of eight neurons over their up rows;
            // else sixteen neurons' rows) once the groups holding them have
            // landed.  A holds 16 (n - 8) of the rows' codes, B x's digits
            // (column p = digit p), so D = 16 * 2^(7p) * xs * (the group's dot
            // with digit p of x), exact in int32; warp w takes the 32-element
            // k-groups of its own x vectors (G = 8 w + 128 kk + j) and adds each
            // group's digit columns, weighted, times the row's group scale.
            if constexpr (WF == kI4) {
                constexpr int kNT = kGated ? 8 : 16;   // neurons per m-tile
                const int g = lane >> 2, tq = lane & 3;
                bool tok = true;
#pragma unroll 1
                for (int n0 = 0; n0 < k && tok; n0 += kNT) {
                    for (int g0 = n0; g0 < min(n0 + kNT, k); g0 += 4) {
                        // this warp waits (bounded) for the group; every lane
                        // then observes the completed phase itself
                        const int gi = (sb + g0) >> 2;
                        const uint32_t par = (gpar >> gi) & 1u;
                        bool ok = true;
                        if (lane == 0 && !mbar_test(&sm.gbar[gi], par)) {
                            const long long t0 = gtimer();
                            for (unsigned it = 1;; ++it) {
                                if (mbar_test(&sm.gbar[gi], par)) break;
                                if ((it & 15) == 0 && gtimer() - t0 > p.wait_ns) { ok = false; break; }
                            }
                        }
                        ok = __shfl_sync(0xffffffffu, ok, 0);
                        if (j0 == 0 && g0 == 0 && warp == 0) prof_put(p, li, 17, gtimer());
                        if (!ok) {
                            if (lane == 0) {
                                set_error(p.err, kDevTimeout);
                                sm.gfail = 1;
                            }
                            tok = false;
                            break;
                        }
                        mbar_test(&sm.gbar[gi], par);   // acquire for this lane
                    }
                    if (!tok) break;
                    // this lane's rows g and g + 8 of the tile (rows past the
                    // round's last neuron read its last slot; never stored)
                    const int na = n0 + g, nb = kGated ? na : n0 + g + 8;
                    const uint8_t *ra = stg + size_t(sb + min(na, k - 1)) * sstr;
                    const uint8_t *rbw = kGated ? ra + p.wrow : stg + size_t(sb + min(nb, k - 1)) * sstr;
                    // this lane's digit columns 2 tq and 2 tq + 1: weights 2^-7p / (16 xs)
                    const float dw0 = tq < 3 ? ldexpf(1.f, -14 * tq - 4) / xs : 0.f;
                    const float dw1 = tq < 2 ? ldexpf(1.f, -14 * tq - 11) / xs : 0.f;
                    float accA = 0.f, accB = 0.f;
#pragma unroll
                    for (int kk = 0; kk < MAXVW; ++kk) {
#pragma unroll 2
                        for (int j = 0; j < 8; ++j) {
                            const int G = 8 * warp + 128 * kk + j;
                            if (G < d / 32) {
                                const uint32_t wa = *reinterpret_cast<const uint32_t *>(ra + G * 16 + 4 * tq);
                                const uint32_t wb = *reinterpret_cast<const uint32_t *>(rbw + G * 16 + 4 * tq);
                                const uint2 bx = reinterpret_cast<const uint2 *>(xp)[(G * 8 + g) * 4 + tq];
                                uint32_t ae, ao, be, bo;
                                i4x8_to_s8(wa, ae, ao);
                                i4x8_to_s8(wb, be, bo);
                                int dd[4];
                                imma16832(dd, ae, be, ao, bo, bx.x, bx.y);
                                const float sa = __half2float(*reinterpret_cast<const __half *>(ra + d / 2 + 2 * G));
                                const float sbw = __half2float(*reinterpret_cast<const __half *>(rbw + d / 2 + 2 * G));
                                accA = fmaf(sa, fmaf(i22_to_f(dd[0]), dw0, i22_to_f(dd[1]) * dw1), accA);
                                accB = fmaf(sbw, fmaf(i22_to_f(dd[2]), dw0, i22_to_f(dd[3]) * dw1), accB);
                            }
                        }
                    }
                    // the digit columns sit in the four lanes of a quad
                    accA += __shfl_xor_sync(0xffffffffu, accA, 1);
                    accB += __shfl_xor_sync(0xffffffffu, accB, 1);
                    accA += __shfl_xor_sync(0xffffffffu, accA, 2);
                    accB += __shfl_xor_sync(0xffffffffu, accB, 2);
                    if (tq == 0) {
                        if constexpr (kGated) {
                            if (na < k) {
                                sm.red[rb][warp][2 * na] = accA;
                                sm.red[rb][warp][2 * na + 1] = accB;
                            }
                        } else {
                            if (na < k) {
                                sm.red[rb][warp][2 * na] = accA;
                                sm.red[rb][warp][2 * na + 1] = 0.f;
                            }
                            if (nb < k) {
                                sm.red[rb][warp][2 * nb] = accB;
                                sm.red[rb][warp][2 * nb + 1] = 0.f;
                            }
                        }
                    }
                }
            } else
            // other formats: four neurons at a time as each group lands; after
            // the reduction lanes 4q .. 4q + 3 hold value q
#pragma unroll 1
            for (int g0 = 0; g0 < k; g0 += 4) {
                {
                    // this warp waits (bounded) for the group; every lane then
                    // observes the completed phase itself
                    const int g = (sb + g0) >> 2;
                    const uint32_t par = (gpar >> g) & 1u;
                    bool ok = true;
                    if (lane == 0 && !mbar_test(&sm.gbar[g], par)) {
                        const long long t0 = gtimer();
                        for (unsigned it = 1;; ++it) {
                            if (mbar_test(&sm.gbar[g], par)) break;
                            if ((it & 15) == 0 && gtimer() - t0 > p.wait_ns) { ok = false; break; }
                        }
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (j0 == 0 && g0 == 0 && warp == 0) prof_put(p, li, 17, gtimer());
                    if (!ok) {
                        if (lane == 0) {
                            set_error(p.err, kDevTimeout);
                            sm.gfail = 1;
                        }
                        break;
                    }
                    mbar_test(&sm.gbar[g], par);   // acquire for this lane
                }
                float v[8];
#pragma unroll
                for (int n = 0; n < 4; ++n) {
                    v[2 * n] = 0.f;
                    v[2 * n + 1] = 0.f;
                    if (g0 + n < k) {
                        const uint8_t *slot = stg + size_t(sb + g0 + n) * sstr;
                        v[2 * n] = dot_smem(slot);
                        if (kGated) v[2 * n + 1] = dot_smem(slot + p.wrow);
                    }
                }
                const float ws = warp_transpose_sum(v);
                const int q = 2 * g0 + (lane >> 2);
                if ((lane & 3) == 0 && q < 2 * k) sm.red[rb][warp][q] = ws;
            }
            cta_sync();
            if (sm.gfail) { gok = false; break; }
            gpar ^= rmask;   // every group of the round completed one phase
            gpend &= ~rmask;
            if (tid < 2 * k) {
                float a = 0.f;
                for (int w = 0; w < kConsumerWarps; ++w) a += sm.red[rb][w][tid];
                sm.rsum[tid] = a;
            }
            rb ^= 1;
            cta_sync();
            if (tid < k) {
                const int e = sm.glst[j0 + tid] >> 24;
                sm.rh[tid] = act_h(p.act, sm.rsum[2 * tid] - sm.gc[j0 + tid], sm.rsum[2 * tid + 1]) * sm.route_w[e];
            }
            cta_sync();
            // neurons with h != 0, in list order (every warp forms the same
            // ballot; warp 0 records them)
            const bool nzv = lane < k && sm.rh[lane] != 0.f;
            const unsigned nzm = __ballot_sync(0xffffffffu, nzv);
            if (warp == 0 && nzv) {
                const int pos = nz_total + __popc(nzm & ((1u << lane) - 1u));
                sm.nz[pos] = sm.glst[j0 + lane];
                sm.hz[pos] = sm.rh[lane];
            }
            const int nz_round = __popc(nzm);
            if constexpr (kSpec) {
                // acc += h * W_down row, kAG neurons at a time: their row
                // vectors are loaded before any of them is accumulated
                constexpr int kAG = MAXVW > 1 ? 2 : 4;
#pragma unroll 1
                for (int g0 = 0; g0 < k; g0 += kAG) {
                    float hv[kAG];
                    VW q[kAG][MAXVW];
#pragma unroll
                    for (int j = 0; j < kAG; ++j) {
                        hv[j] = g0 + j < k ? sm.rh[g0 + j] : 0.f;
                        const uint8_t *row = stg + size_t(sb + g0 + j) * sstr + p.gu_bytes;
#pragma unroll
                        for (int kk = 0; kk < MAXVW; ++kk) {
                            const int v = tid + kThreads * kk;
                            if (hv[j] != 0.f && v < nvecW) q[j][kk] = *reinterpret_cast<const VW *>(row + v * VBW);
                        }
                    }
#pragma unroll
                    for (int j = 0; j < kAG; ++j) {
                        if (hv[j] == 0.f) continue;
                        const uint8_t *row = stg + size_t(sb + g0 + j) * sstr + p.gu_bytes;
#pragma unroll
                        for (int kk = 0; kk < MAXVW; ++kk) {
                            const int v = tid + kThreads * kk;
                            if (v < nvecW) {
                                float w[EPVW];
                                cvt<WF>(q[j][kk], w);
                                float hs = hv[j];
                                if constexpr (WF == kI4)
                                    hs *= __half2float(*reinterpret_cast<const __half *>(row + d / 2 + (v >> 2) * 2));
#pragma unroll
                                for (int i = 0; i < EPVW; ++i) acc[kk * EPVW + i] = fmaf(hs, w[i], acc[kk * EPVW + i]);
                            }
                        }
                    }
                }
            }
            nz_total += nz_round;
            cta_sync();   // the round's slots are reused by the next batch
        }
        prof_put(p, li, 25, gtimer());
        // not speculative: the W_down rows of the neurons with h != 0, in rounds
        if (gok && !kSpec) {
            const int cap_d = min(kMaxTopK * kMaxStrip, kStageBytes / p.wrow);
            for (int q0 = 0; q0 < nz_total && gok; q0 += cap_d) {
                const int k = min(cap_d, nz_total - q0);
                if (warp == 0) {
                    int nhot = 0;
                    for (int n = lane; n < k; n += 32)
                        nhot += (unsigned(sm.nz[q0 + n]) & kColdBit) ? 0 : 1;
                    nhot = __reduce_add_sync(0xffffffffu, nhot);
                    if (lane == 0) mbar_arrive_tx(&sm.stage_bar, uint32_t(nhot) * p.wrow);
                    __syncwarp();
                    for (int n = lane; n < k; n += 32) {
                        const int en = sm.nz[q0 + n], e = en >> 24;
                        if (unsigned(en) & kColdBit) continue;
                        const unsigned code = unsigned(en) & 0xffffffu;
                        stage_copy(stg + size_t(n) * p.wrow, exs[e]->Wd + size_t(code) * p.wd_stride,
                                   uint32_t(p.wrow), &sm.stage_bar);
                    }
                }
                if (p.hot_k) {
                    for (int n = 0; n < k; ++n) {
                        const int en = sm.nz[q0 + n];
                        if (!(unsigned(en) & kColdBit)) continue;
                        const unsigned idx = unsigned(en) & (kColdBit - 1u);
                        copy_host_rec(stg + size_t(n) * p.wrow, exs[en >> 24]->Wd_cold + size_t(idx) * p.wd_stride,
                                      p.wrow, tid, kThreads);
                    }
                    cta_sync();
                }
                pending = true;
                if (!stage_wait(&sm, p, spar, bci, &cyc_c)) { gok = false; break; }
                pending = false;
                for (int n = 0; n < k; ++n) axpy_smem(stg + size_t(n) * p.wrow, sm.hz[q0 + n]);
                cta_sync();
            }
        }
        if (!gok) break;
        prof_put(p, li, 26, gtimer());
        if (tid == 0 && p.stats) atomicAdd(p.stats + li * 4 + 1, nz_total);
        (void)cc0;

        // ---------------- y: the CTAs' partials summed in fixed point --------
        // This CTA's partial of y as 64-bit fixed-point values at the top of
        // the staging buffer, added into layer l's total by one bulk reduction
        // (integer adds, so the total does not depend on their order); the
        // arrival follows its completion.
        {
            unsigned long long *ys = reinterpret_cast<unsigned long long *>(stg + yoff);
#pragma unroll
            for (int k = 0; k < MAXVW; ++k) {
                const int v = tid + kThreads * k;
                if (v < nvecW) {
#pragma unroll
                    for (int i = 0; i < EPVW; i += 2)
                        *reinterpret_cast<ulonglong2 *>(ys + v * EPVW + i) =
                            make_ulonglong2(fix_q(acc[k * EPVW + i], p.err), fix_q(acc[k * EPVW + i + 1], p.err));
                }
            }
            fence_proxy_async_smem();
        }
        cta_sync();
        if (tid == 0) {
            fence_proxy_async_global();
            bulk_reduce_add_u64(p.yfix + size_t(l & 1) * d, stg + yoff, uint32_t(d) * 8u);
            bulk_wait_all();
            fence_proxy_async_global();
        }
        prof_put(p, li, 3, gtimer());
        grid_arrive(p, epoch);
        // the next layer's V rows and first U piece (dense) start moving once
        // this CTA has arrived (the arrival's release would otherwise wait
        // for these copies)
        const bool next = l + 1 < l1;
        if (next && warp == 0 && vsm) stage_next_dense(l + 1);
        if (next && vsm) vpend = true;
        if (next && vsm && ns > 0) {
            staged_early = pending = true;
            upart2 = ufirst < u_round0;
        }
        if (!grid_wait(&sm, p, epoch, bci, &cyc_bar)) break;
        prof_put(p, li, 4, gtimer());
    }
    // an early exit may leave one staging round in flight: let it land
    // (bounded) so no bulk copy writes this CTA's shared memory after exit
    if (tid == 0) {
        const long long t0 = gtimer();
        // a U round staged in two pieces whose second piece was never issued:
        // arrive for it, so the phase completes when the first piece lands
        if (upart2) mbar_arrive(&sm.stage_bar);
        if (pending)
            while (!mbar_test(&sm.stage_bar, spar) && gtimer() - t0 < p.wait_ns) {
            }
        if (vpend)
            while (!mbar_test(&sm.vbar, vpar) && gtimer() - t0 < p.wait_ns) {
            }
        for (int g = 0; g < kIssue / 4; ++g)
            if ((gpend >> g) & 1u)
                while (!mbar_test(&sm.gbar[g], (gpar >> g) & 1u) && gtimer() - t0 < p.wait_ns) {
                }
    }
}

// One instantiation per (weight format, predictor format, d_model class,
// layer kind); each per-format translation unit instantiates its own set.
template <int WF, int PF, int DMAX, int MODE>
cudaError_t launch_one(const DecodeParams &p, cudaStream_t st, bool query, int *blocks)
{
    void *fn = (void *)decode_kernel<WF, PF, DMAX, MODE>;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kStageBytes);
    if (e != cudaSuccess) return e;
    if (query) return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks, fn, kThreads, kStageBytes);
    void *args[] = {const_cast<DecodeParams *>(&p)};
    return cudaLaunchCooperativeKernel(fn, dim3(p.S), dim3(kThreads), args, kStageBytes, st);
}

template <int WF, int PF, int DMAX>
cudaError_t launch_mode(int mode, const DecodeParams &p, cudaStream_t st, bool query, int *blocks)
{
    switch (mode) {
    case kModeSpec: return launch_one<WF, PF, DMAX, kModeSpec>(p, st, query, blocks);
    case kModeGated | kModeSpec: return launch_one<WF, PF, DMAX, kModeGated | kModeSpec>(p, st, query, blocks);
    case kModeGated: return launch_one<WF, PF, DMAX, kModeGated>(p, st, query, blocks);
    case kModeMoE | kModeSpec: return launch_one<WF, PF, DMAX, kModeMoE | kModeSpec>(p, st, query, blocks);
    case kModeMoE | kModeGated | kModeSpec:
        return launch_one<WF, PF, DMAX, kModeMoE | kModeGated | kModeSpec>(p, st, query, blocks);
    case kModeMoE | kModeGated: return launch_one<WF, PF, DMAX, kModeMoE | kModeGated>(p, st, query, blocks);
    case kModePred: return launch_one<WF, PF, DMAX, kModePred>(p, st, query, blocks);
    case kModePred | kModeMoE: return launch_one<WF, PF, DMAX, kModePred | kModeMoE>(p, st, query, blocks);
    default: return cudaErrorInvalidValue;
    }
}

// d_model classes: the register arrays of x hold ceil(d / (elements per
// vector * threads)) vectors per thread, so two classes cover d <= 8192
// (d <= 4096 for fp32).
template <int WF, int PF>
cudaError_t launch_fmt(int d, int mode, const DecodeParams &p, cudaStream_t st, bool query, int *blocks)
{
    constexpr int kSmall = (WF == kF32 || PF == kF32) ? 2048 : 4096;
    if (d <= kSmall) return launch_mode<WF, PF, kSmall>(mode, p, st, query, blocks);
    if (d <= 2 * kSmall) return launch_mode<WF, PF, 2 * kSmall>(mode, p, st, query, blocks);
    return cudaErrorInvalidValue;
}

}  // namespace
}  // namespace pi
