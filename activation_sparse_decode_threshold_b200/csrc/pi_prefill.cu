// pi_prefill.cu -- dense multi-token prefill on the sm_100a tensor cores.
//
// PowerInfer-2 runs prefill as large dense neuron clusters ("Neuron-cluster
// heterogeneous computing", citnews.com.cn article): with many tokens almost
// every neuron fires, so the FFN is a real dense contraction and goes to the
// tensor cores.  Per layer:
//
//   k_norm_route   x = RMSNorm(r) per token (fp32), an fp16 copy for the MMA,
//                  MoE router logits (fp32) and top-2 with renormalised weights
//   k_sort         tokens grouped by expert (counting sort, ascending token
//                  order inside each expert: deterministic)
//   k_gemm<GU>     per expert: [tokens x d] x [d x 2F] -> gate and up for 128
//                  neurons per CTA tile (their rows interleaved so one TMEM
//                  column pair holds a neuron's g and u), activation fused in
//                  the epilogue: H = act(g - c, u) (fp16)
//   k_gemm<DOWN>   per expert: H [tokens x F] x W_down^T [F x d], split over
//                  K into fp32 partials (W_down stored neuron-major is the
//                  MN-major operand)
//   k_combine      y = sum over the token's experts in ascending expert index
//                  of w * (sum of the K-split partials, fixed order); r += y
//
// GEMM tiles: up to 256 list positions (two 128-row halves) x 256 weight rows
// x 64 per stage.  The activation halves arrive by 2-D tensor-map loads in
// the 128-byte swizzle; the weight tile is written into shared memory by the
// CTA's threads (INT4 weights dequantised to fp16 on the way), in the same
// swizzle for the K-major gate/up weights and in the canonical no-swizzle
// core-matrix layout (8 k-rows x 16 bytes) for the MN-major W_down, once per
// stage for both halves.  One elected thread issues tcgen05.mma (kind::f16,
// M = 128, N = 256, fp32 accumulators in TMEM, one per half) four K=16 steps
// per stage and half, and tcgen05.commit on a per-stage mbarrier frees the
// stage.  Three stages.  Every wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdio>
#include <cstring>
#include <vector>

#include "pi_prefill.h"

namespace pi {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, NSTAGE = 3;
constexpr int kHalves = 2;                        // 128-row halves of a CTA's rows (one accumulator each)
constexpr int kTileRows = kHalves * BM;
constexpr int kProducerWarps = 16, kProducers = 32 * kProducerWarps;
constexpr int kRI = BN * 4 / kProducers;          // INT4 items (16 weights) per producer thread per stage
constexpr int kEpiCols = BN / (kProducerWarps / 4); // accumulator columns per epilogue warp
constexpr int kGemmThreads = kProducers + 64;    // + the MMA warp + the INT4 raw loader warp
constexpr int kLag = 1;                          // stages between issuing a stage's copies and publishing it
constexpr int kATileBytes = BM * BK * 2;          // 16 KB
constexpr int kBTileBytes = BN * BK * 2;          // 32 KB
constexpr int kStageBytes = kHalves * kATileBytes + kBTileBytes;   // 64 KB
constexpr int kGemmSmem = NSTAGE * kStageBytes + 1024;
// INT4 weights reach shared memory by tensor-map loads, raw, kRawSlots K steps
// ahead of their dequantisation: a gate/up stage is 256 rows x 32 bytes of
// nibbles, a down stage 64 k-rows x 128 bytes; the gate/up scales come in
// chunks of four K steps (256 rows x 16 bytes), the down scales per step
// (64 k-rows x 16 bytes)
constexpr int kRawSlots = 3;
constexpr int kRawBytes = 8192;
constexpr int kScaleChunk = 4096;
constexpr int kGemmSmemI4 = kGemmSmem + kRawSlots * kRawBytes + 2 * kScaleChunk;
constexpr int kTmemCols = kHalves * BN;           // 512: the whole tensor memory (one CTA per SM)
constexpr int kSplitK = 4;                        // K splits of the down GEMM

enum GemmKind { kGU = 0, kDOWN = 1 };

struct PrefillExpert {
    const uint8_t *Wgu;   // F neuron records rec_bytes apart (gate row, then up row when gated)
    const uint8_t *Wd;    // F rows of wrow bytes (W_down columns)
    const float *c;       // F biases
};

struct GemmParams {
    PrefillExpert ex[kMaxExperts];
    int E, d, F, gated, act, wrow, rec_bytes, wd_stride;
    const int32_t *e_off;     // [E + 1] first list position of each expert
    const int32_t *e_tok;     // [2T] token of each list position
    void *H;                  // [2T x F] activations per list position (same type)
    float *Ypart;             // [kSplitK x 2T x d] down partials
    int rows_cap;             // 2T
    int *err;
    long long wait_ns;        // bound on every mbarrier wait
    int debug_flags;          // PI_DEBUG_STALL_PREFILL: one producer withholds its first arrival
    // A operand: rows of list positions (normalised inputs sorted by expert for
    // the gate/up GEMM, H for the down GEMM), 64 x 128 boxes with 128-byte swizzle
    alignas(64) CUtensorMap tmA;
    // INT4 weights of each expert, as bytes: gate/up nibbles (boxes of 32 bytes
    // x {gate, up} x 128 neurons) and scales (16 bytes x {gate, up} x 128), or
    // down nibbles (128 bytes x 64 k-rows, 128-byte swizzle) and scales (16 x 64)
    alignas(64) CUtensorMap tmW[kMaxExperts];
    alignas(64) CUtensorMap tmS[kMaxExperts];
};

// ---------------------------------------------------------------------------
// PTX helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t s2u(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t *b, unsigned count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(s2u(b)), "r"(count) : "memory");
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
__device__ __forceinline__ long long gtimer()
{
    long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// bounded wait; false (and the error word set) when it runs out
__device__ bool mbar_wait(uint64_t *b, uint32_t parity, int *err, long long wait_ns)
{
    if (mbar_test(b, parity)) return true;
    const long long t0 = gtimer();
    for (unsigned it = 1;; ++it) {
        if (mbar_test(b, parity)) return true;
        if ((it & 15) == 0 && gtimer() - t0 > wait_ns) {
            atomicCAS(err, 0, int(kDevTimeout));
            return false;
        }
    }
}
__device__ __forceinline__ void cp_async16(void *dst, const void *src, bool pred)
{
    const int n = pred ? 16 : 0;   // zero-fill when out of range
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s2u(dst)), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void mbar_arrive_tx(uint64_t *b, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(s2u(b)), "r"(bytes) : "memory");
}
// 2-D tiled TMA load of box (x, y) into shared memory, completion on `bar`
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(s2u(dst)), "l"(map), "r"(x), "r"(y), "r"(s2u(bar))
        : "memory");
}
// 3-D tiled TMA load of box (x, y, z) into shared memory, completion on `bar`
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int x, int y, int z, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
        ::"r"(s2u(dst)), "l"(map), "r"(x), "r"(y), "r"(z), "r"(s2u(bar))
        : "memory");
}
// shared-memory matrix descriptor of a K-major tile with 128-byte swizzle (rows
// of 128 bytes, 8-row groups 1024 bytes apart, as the tensor-map load writes
// them); the start address moves by 32 bytes per 16-element K step
__device__ __forceinline__ uint64_t make_sdesc_sw128(uint32_t saddr)
{
    uint64_t d = 0;
    d |= uint64_t((saddr >> 4) & 0x3fff);
    d |= uint64_t(1) << 16;             // leading byte offset (unused with this layout)
    d |= uint64_t(1024 >> 4) << 32;     // stride byte offset: 8 rows x 128 bytes
    d |= uint64_t(1) << 46;             // descriptor version
    d |= uint64_t(2) << 61;             // 128-byte swizzle
    return d;
}
// shared-memory matrix descriptor: canonical layout without swizzle; start,
// leading (K direction) and stride (M/N direction) byte offsets in 16-byte
// units; descriptor version 1
__device__ __forceinline__ uint64_t make_sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    uint64_t d = 0;
    d |= uint64_t((saddr >> 4) & 0x3fff);
    d |= uint64_t((lbo >> 4) & 0x3fff) << 16;
    d |= uint64_t((sbo >> 4) & 0x3fff) << 32;
    d |= uint64_t(1) << 46;
    return d;
}
// instruction descriptor: f16 A and B, f32 accumulate, M = m (128 or 64), N = 256
__device__ __forceinline__ uint32_t make_idesc(bool b_mn_major, bool bf16, int m = BM)
{
    uint32_t i = 0;
    i |= 1u << 4;                        // D format: f32
    i |= (bf16 ? 1u : 0u) << 7;          // A: f16 / bf16
    i |= (bf16 ? 1u : 0u) << 10;         // B: same type as A
    i |= 0u << 15;                       // A K-major
    i |= (b_mn_major ? 1u : 0u) << 16;   // B K-major / MN-major
    i |= uint32_t(BN >> 3) << 17;
    i |= uint32_t(m >> 4) << 24;
    return i;
}
__device__ __forceinline__ void umma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, bool acc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc ? 1u : 0u)
        : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(s2u(bar)) : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float *v)
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// byte offset of 16-byte chunk `kc` (0..7) of row `row` of a K-major tile
// with 128-byte rows in the 128-byte swizzle (the chunk index XOR the row
// mod 8, 8-row groups 1024 bytes apart), the layout a SWIZZLE_128B
// tensor-map load writes; 8 consecutive rows of one chunk fall in 8
// different bank groups
__device__ __forceinline__ uint32_t sw128_off(int row, int kc)
{
    return uint32_t((row >> 3) * 1024 + (row & 7) * 128 + ((kc ^ (row & 7)) << 4));
}
// byte offset of the 16-byte chunk holding n = 8*ng .. 8*ng+7 of k-row `k`
// in an MN-major tile (core matrices: 8 k-rows x 8 n-values)
__device__ __forceinline__ uint32_t mnmaj_off(int ng, int k)
{
    return uint32_t(ng * (BK / 8 * 128) + (k >> 3) * 128 + (k & 7) * 16);
}

// 16 INT4 weights (8 bytes of nibbles, low nibble = even element) with their
// group scale -> 16 fp16 values s * (n - 8), on the integer and half pipes: a
// nibble n placed in the fraction of the half 1024.0 (byte permutes put each
// nibble under a 0x64 exponent byte) gives 1024 + n exactly, subtracting
// 1032 gives n - 8 exactly, and the product with s is rounded once, as a
// rounding of the exact s * (n - 8) to fp16.
__device__ __forceinline__ void dequant16(uint2 q, __half s, uint4 &lo, uint4 &hi)
{
    const __half2 s2 = __halves2half2(s, s);
    const __half2 off = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));   // 1032
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const uint32_t w = i == 0 ? q.x : q.y;
        const uint32_t ev = w & 0x0F0F0F0Fu, od = (w >> 4) & 0x0F0F0F0Fu;   // even / odd elements
        const uint32_t p01 = __byte_perm(ev, od, 0x5140), p23 = __byte_perm(ev, od, 0x7362);
        const uint32_t bits[4] = {__byte_perm(p01, 0x64646464u, 0x4140), __byte_perm(p01, 0x64646464u, 0x4342),
                                  __byte_perm(p23, 0x64646464u, 0x4140), __byte_perm(p23, 0x64646464u, 0x4342)};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            __half2 h = *reinterpret_cast<const __half2 *>(&bits[m]);
            h = __hmul2(__hsub2(h, off), s2);
            o[4 * i + m] = *reinterpret_cast<const uint32_t *>(&h);
        }
    }
    lo = make_uint4(o[0], o[1], o[2], o[3]);
    hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// ---------------------------------------------------------------------------
// GEMM kernel.  Warps 0-15 produce stages (cp.async for 16-bit operands, INT4
// weights through registers seven stages ahead and dequantised into the tile),
// warp 16 issues the MMAs from one thread, and warps 0-15 run the epilogue
// once the accumulator is complete.  Stage s is published on full[s] (every
// producer thread arrives after its copies landed and a proxy fence) and
// freed on empty[s] by tcgen05.commit.
// ---------------------------------------------------------------------------
template <int W> struct Elem { using T = __half; };
template <> struct Elem<1> { using T = __nv_bfloat16; };
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ __half from_f<__half>(float x) { return __float2half_rn(x); }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ void mbar_arrive(uint64_t *b)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(s2u(b)) : "memory");
}

template <int KIND, int W>
__global__ void __launch_bounds__(kGemmThreads, 1) k_gemm(const __grid_constant__ GemmParams p)
{
    constexpr bool I4 = W == 2;
    using AT = typename Elem<W>::T;
    AT *Hbuf = reinterpret_cast<AT *>(p.H);
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full[NSTAGE], afull[NSTAGE], empty[NSTAGE], done;
    __shared__ uint64_t rbar[kRawSlots], rfree[kRawSlots];   // INT4 raw ring: landed / consumed
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile int abort_sh;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int d = p.d, F = p.F;
    // tile coordinates: blockIdx.x = N tile, blockIdx.y = M tile (up to 256
    // list positions of one expert) over all experts, blockIdx.z = K split
    // (down GEMM)
    int e = -1, mrow0 = 0;
    {
        int acc = 0;
        for (int x = 0; x < p.E; ++x) {
            const int cnt = p.e_off[x + 1] - p.e_off[x];
            const int tiles = (cnt + kTileRows - 1) / kTileRows;
            if (int(blockIdx.y) < acc + tiles) {
                e = x;
                mrow0 = p.e_off[x] + (int(blockIdx.y) - acc) * kTileRows;
                break;
            }
            acc += tiles;
        }
    }
    if (e < 0) return;   // uniform: no tile for this CTA
    const int mrow_end = p.e_off[e + 1];
    const int nh = mrow_end - mrow0 > BM ? 2 : 1;   // halves holding rows of this expert
    // a second half of at most 64 rows takes an M = 64 MMA: its accumulator
    // row 16 q + i sits in TMEM lane 32 q + i (i < 16) of the half's columns
    const bool h1_m64 = nh == 2 && mrow_end - mrow0 <= BM + 64;
    const PrefillExpert ex = p.ex[e];
    const int K = KIND == kGU ? d : F;
    const int nk_all = K / BK;
    const int ksplit = KIND == kGU ? 1 : kSplitK;
    const int kt0 = int((long long)blockIdx.z * nk_all / ksplit), kt1 = int((long long)(blockIdx.z + 1) * nk_all / ksplit);
    const int nk = kt1 - kt0;
    const int n0 = blockIdx.x * BN;   // GU: B-row 2j/2j+1 = gate/up of neuron n0/2 + j

    if (tid == 0) {
        for (int s = 0; s < NSTAGE; ++s) {
            mbar_init(&full[s], kProducers);
            mbar_init(&afull[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < kRawSlots; ++s) {
            mbar_init(&rbar[s], 1);
            mbar_init(&rfree[s], kProducers);
        }
        mbar_init(&done, 1);
        abort_sh = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kProducerWarps) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(s2u(&tmem_base_sh)), "r"(kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = tmem_base_sh;

    uint8_t *const raw = smem + NSTAGE * kStageBytes;
    uint8_t *const scl = raw + kRawSlots * kRawBytes;
    auto issue_raw = [&](int q) {   // the loader warp: stage q of this CTA's K range
        const int slot = q % kRawSlots, kt = kt0 + q;
        uint8_t *dst = raw + slot * kRawBytes;
        if constexpr (KIND == kGU) {
            const int G = p.gated ? 2 : 1;
            const bool sc = q == 0 || (kt & 3) == 0;
            mbar_arrive_tx(&rbar[slot], uint32_t(G * (BN / 2) * (BK / 2) + (sc ? G * (BN / 2) * 16 : 0)));
            tma_load_3d(dst, &p.tmW[e], kt * (BK / 2), 0, n0 / 2, &rbar[slot]);
            if (sc)
                tma_load_3d(scl + ((kt >> 2) & 1) * kScaleChunk, &p.tmS[e], d / 2 + (kt >> 2) * 16, 0, n0 / 2,
                            &rbar[slot]);
        } else {
            mbar_arrive_tx(&rbar[slot], uint32_t(kRawBytes + BK * 16));
            tma_load_2d(dst, &p.tmW[e], n0 / 2, kt * BK, &rbar[slot]);
            tma_load_2d(scl + slot * (BK * 16), &p.tmS[e], d / 2 + n0 / 16, kt * BK, &rbar[slot]);
        }
    };

    if (warp < kProducerWarps) {
        // ------------------------------ producers ------------------------------
        const int pt = tid;   // 0 .. 255
        // Chunk-to-lane mapping of the B tile: a warp covers 8 consecutive
        // rows x 4 consecutive 16-byte chunks, so its global reads are whole
        // 32-byte sectors and its shared stores are four 128-byte runs (no bank
        // conflicts beyond the minimum).  The A tile comes by tensor-map load.
        auto issue_async = [&](int kt, int s) {
            uint8_t *A = smem + s * kStageBytes;
            uint8_t *B = A + kHalves * kATileBytes;
            const int k0 = kt * BK;
            if (pt == 0) {
                // A: one or two halves of 128 list positions x 64 elements; rows
                // past the expert's are loaded too and their results discarded,
                // rows past the buffer read 0
                mbar_arrive_tx(&afull[s], uint32_t(nh * kATileBytes));
                tma_load_2d(A, &p.tmA, k0, mrow0, &afull[s]);
                if (nh > 1) tma_load_2d(A + kATileBytes, &p.tmA, k0, mrow0 + BM, &afull[s]);
            }
            if constexpr (!I4) {
                if constexpr (KIND == kGU) {
#pragma unroll
                    for (int i = 0; i < BN * (BK / 8) / kProducers; ++i) {   // 256 rows x 8 chunks, K-major
                        const int c = pt + kProducers * i, rest = c >> 5;
                        const int row = (rest & 31) * 8 + (c & 7), kc = (rest >> 5) * 4 + ((c >> 3) & 3);
                        const int nn = n0 / 2 + (row >> 1);
                        const bool ok = nn < F && (p.gated || (row & 1) == 0);
                        const uint8_t *rec = ex.Wgu + size_t(ok ? nn : 0) * p.rec_bytes + ((row & 1) ? p.wrow : 0);
                        cp_async16(B + sw128_off(row, kc), rec + (k0 + kc * 8) * 2, ok);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < BK * (BN / 8) / kProducers; ++i) {   // 64 k-rows x 32 chunks, MN-major
                        const int c = pt + kProducers * i, rest = c >> 5;
                        const int k = (rest & 7) * 8 + (c & 7), ng = (rest >> 3) * 4 + ((c >> 3) & 3);
                        const uint8_t *row = ex.Wd + size_t(k0 + k) * p.wd_stride + (n0 + ng * 8) * 2;
                        cp_async16(B + mnmaj_off(ng, k), row, true);
                    }
                }
            }
            if constexpr (!I4) cp_async_commit();
        };
        // INT4: raw stages reach shared memory by tensor-map loads (the loader
        // warp below), kRawSlots stages in flight: rbar[q % kRawSlots]
        // completes stage q; every producer arrives on rfree[q % kRawSlots]
        // once it has dequantised stage q, so the slot can take stage
        // q + kRawSlots.  Gate/up item c: row c / 4 of the tile, 16 elements
        // (c % 4) of the K step: a warp reads 256 contiguous raw bytes and
        // writes four 128-byte runs.  Down item: W_down row k (8 per warp) and
        // 16 output columns, the raw rows in 128-byte swizzle so 8 rows of one
        // column chunk fall in 8 bank groups.
        auto dequant_stage = [&](int q, int s) {
            const int slot = q % kRawSlots, kt = kt0 + q;
            const uint8_t *rw = raw + slot * kRawBytes;
            uint8_t *B = smem + s * kStageBytes + kHalves * kATileBytes;
#pragma unroll
            for (int i = 0; i < kRI; ++i) {
                const int c = pt + kProducers * i;
                uint2 qv = make_uint2(0u, 0u);
                unsigned short sv = 0;
                if constexpr (KIND == kGU) {
                    const int row = c >> 2, q16 = c & 3;
                    const bool ok = p.gated || (row & 1) == 0;
                    const int rr = p.gated ? row : row >> 1;
                    if (ok) {
                        qv = *reinterpret_cast<const uint2 *>(rw + rr * (BK / 2) + q16 * 8);
                        sv = *reinterpret_cast<const unsigned short *>(
                            scl + ((kt >> 2) & 1) * kScaleChunk + rr * 16 + ((kt & 3) * 2 + (q16 >> 1)) * 2);
                    }
                    uint4 lo, hi;
                    dequant16(qv, __ushort_as_half(sv), lo, hi);
                    *reinterpret_cast<uint4 *>(B + sw128_off(row, 2 * q16)) = lo;
                    *reinterpret_cast<uint4 *>(B + sw128_off(row, 2 * q16 + 1)) = hi;
                } else {
                    const int rest = c >> 5;
                    const int k = (rest & 7) * 8 + (c & 7), g16 = (rest >> 3) * 4 + ((c >> 3) & 3);
                    qv = *reinterpret_cast<const uint2 *>(rw + k * 128 + (((g16 >> 1) ^ (k & 7)) << 4) + (g16 & 1) * 8);
                    sv = *reinterpret_cast<const unsigned short *>(scl + slot * (BK * 16) + k * 16 + (g16 >> 1) * 2);
                    uint4 lo, hi;
                    dequant16(qv, __ushort_as_half(sv), lo, hi);
                    *reinterpret_cast<uint4 *>(B + mnmaj_off(2 * g16, k)) = lo;
                    *reinterpret_cast<uint4 *>(B + mnmaj_off(2 * g16 + 1, k)) = hi;
                }
            }
        };
        // publish stage `j`: its copies have landed (cp.async group), make
        // them and the dequantised stores visible to the tensor core, arrive
        // (testing aid: with PI_DEBUG_STALL_PREFILL, producer 0 of the first
        // gate/up CTA never arrives for its first stage, so the MMA warp's
        // bounded wait runs out before any MMA is issued)
        const bool withhold = (p.debug_flags & 2) && KIND == kGU && pt == 0 &&
                              blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0;
        auto publish = [&](int j) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            if (!(withhold && j == 0)) mbar_arrive(&full[j % NSTAGE]);
        };
        int j = 0;
        bool stop = nk == 0;
        while (!stop) {
            const int s = j % NSTAGE;
            if (j >= NSTAGE) {
                // the MMAs of step j - NSTAGE read this stage
                if (!mbar_wait(&empty[s], uint32_t(((j - NSTAGE) / NSTAGE) & 1), p.err, p.wait_ns)) abort_sh = 1;
            }
            if (abort_sh) break;
            issue_async(kt0 + j, s);
            if constexpr (I4) {
                if (!mbar_wait(&rbar[j % kRawSlots], uint32_t((j / kRawSlots) & 1), p.err, p.wait_ns)) {
                    abort_sh = 1;
                    break;
                }
                dequant_stage(j, s);
                mbar_arrive(&rfree[j % kRawSlots]);
                publish(j);
            } else if (j >= kLag) {
                cp_async_wait<kLag>();
                publish(j - kLag);
            }
            if (++j >= nk) stop = true;
        }
        // drain: publish the stages still in flight (all of them on abort too,
        // so that no copy is outstanding at exit)
        if constexpr (!I4) {
            cp_async_wait<0>();
            for (int q = max(0, j - kLag); q < j; ++q) publish(q);
        }
        // no tensor-map load may still be writing this CTA's shared memory at
        // exit: the issuing thread waits (bounded) for the last loads it issued
        if (pt == 0) {
            for (int q = max(0, j - NSTAGE); q < j; ++q)
                mbar_wait(&afull[q % NSTAGE], uint32_t((q / NSTAGE) & 1), p.err, p.wait_ns);
        }
        // epilogue: wait for the accumulator
        if (nk > 0 && !abort_sh && !mbar_wait(&done, 0u, p.err, p.wait_ns)) abort_sh = 1;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const int col0 = kEpiCols * (warp >> 2);
        for (int h = 0; h < nh; ++h) {
            const bool m64 = h == 1 && h1_m64;
            const int lr = mrow0 + h * BM + (m64 ? 16 : 32) * (warp & 3) + lane;
            const bool valid = (!m64 || lane < 16) && lr < mrow_end && !abort_sh;
            if (KIND == kDOWN && nk == 0) {
                // an empty K range still owns its partial: zeros
                if (valid) {
                    float *dst = p.Ypart + (size_t(blockIdx.z) * p.rows_cap + lr) * d + n0 + col0;
                    for (int j2 = 0; j2 < kEpiCols; j2 += 4) *reinterpret_cast<float4 *>(dst + j2) = make_float4(0.f, 0.f, 0.f, 0.f);
                }
                continue;
            }
            if (abort_sh) break;
            for (int cc = 0; cc < kEpiCols; cc += 16) {
                float v[16];
                tmem_ld16(tmem + (uint32_t(32 * (warp & 3)) << 16) + uint32_t(h * BN + col0 + cc), v);
                if (!valid) continue;
                if constexpr (KIND == kGU) {
                    // columns 2j, 2j+1 = gate, up of neuron n0/2 + (col0 + cc)/2 + j
                    const int nb = n0 / 2 + (col0 + cc) / 2;
                    AT hv[8];
#pragma unroll
                    for (int j2 = 0; j2 < 8; ++j2) {
                        const int nn = nb + j2;
                        const float g = v[2 * j2] - (nn < F ? __ldg(ex.c + nn) : 0.f);
                        const float u = v[2 * j2 + 1];
                        const float gp = g > 0.f ? g : 0.f;
                        const float hh = p.act == 0 ? gp : (p.act == 1 ? gp * u : gp * (u > 0.f ? u : 0.f));
                        hv[j2] = from_f<AT>(hh);
                    }
                    if (nb + 8 <= F)
                        *reinterpret_cast<uint4 *>(Hbuf + size_t(lr) * F + nb) = *reinterpret_cast<uint4 *>(hv);
                } else {
                    float *dst = p.Ypart + (size_t(blockIdx.z) * p.rows_cap + lr) * d + n0 + col0 + cc;
#pragma unroll
                    for (int j2 = 0; j2 < 16; j2 += 4)
                        *reinterpret_cast<float4 *>(dst + j2) = make_float4(v[j2], v[j2 + 1], v[j2 + 2], v[j2 + 3]);
                }
            }
        }
    } else if (warp == kProducerWarps && nk > 0) {
        // ------------------------------ MMA issue ------------------------------
        if (lane == 0) {
            const uint32_t idesc = make_idesc(KIND == kDOWN, W == 1);
            const uint32_t idesc1 = h1_m64 ? make_idesc(KIND == kDOWN, W == 1, 64) : idesc;
            int issued = 0;
            for (int j = 0; j < nk; ++j) {
                const int s = j % NSTAGE;
                if (!mbar_wait(&full[s], uint32_t((j / NSTAGE) & 1), p.err, p.wait_ns) ||
                    !mbar_wait(&afull[s], uint32_t((j / NSTAGE) & 1), p.err, p.wait_ns)) { abort_sh = 1; break; }
                if (abort_sh) break;
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t a0 = s2u(smem + s * kStageBytes), b0 = a0 + kHalves * kATileBytes;
#pragma unroll
                for (int ks = 0; ks < BK / 16; ++ks) {
                    // the weight tile's K step feeds each half's accumulator
                    const uint64_t bd = KIND == kGU ? make_sdesc_sw128(b0 + ks * 32)
                                                    : make_sdesc(b0 + ks * 256, 128, BK / 8 * 128);
                    umma(tmem, make_sdesc_sw128(a0 + ks * 32), bd, idesc, j > 0 || ks > 0);
                    if (nh > 1)
                        umma(tmem + uint32_t(BN), make_sdesc_sw128(a0 + kATileBytes + ks * 32), bd, idesc1, j > 0 || ks > 0);
                }
                umma_commit(&empty[s]);
                issued = j + 1;
            }
            // the accumulator is complete when every issued MMA is: one more
            // commit (it tracks all earlier MMAs of this thread)
            umma_commit(&done);
            if (issued < nk) {
                // aborted: let the issued MMAs finish (bounded) before TMEM is freed
                mbar_wait(&done, 0u, p.err, p.wait_ns);
            }
        }
        __syncwarp();
    }
    if (I4 && warp == kProducerWarps + 1 && lane == 0) {
        // ------------------------------ INT4 raw loader ------------------------------
        // stage q's nibbles and scales start moving as soon as its slot is free
        int issued = 0;
        for (int q = 0; q < nk && !abort_sh; ++q) {
            if (q >= kRawSlots &&
                !mbar_wait(&rfree[q % kRawSlots], uint32_t(((q - kRawSlots) / kRawSlots) & 1), p.err, p.wait_ns)) {
                abort_sh = 1;
                break;
            }
            issue_raw(q);
            issued = q + 1;
        }
        // no tensor-map load may still be writing this CTA's shared memory at
        // exit: the last loads issued land (bounded)
        for (int q = max(0, issued - kRawSlots); q < issued; ++q)
            mbar_wait(&rbar[q % kRawSlots], uint32_t((q / kRawSlots) & 1), p.err, p.wait_ns);
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == kProducerWarps)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
}

// ---------------------------------------------------------------------------
// Per-token kernels
// ---------------------------------------------------------------------------
struct TokenParams {
    float *resid;             // [T x d]
    void *X16;                // [T x d], fp16 or bf16 (x_bf16)
    int x_bf16;
    const __half *router;     // [E x d] or null
    int d, E, T, top_k;
    float eps;
    int32_t *route_e;         // [T x 2]
    float *route_w;           // [T x 2]
    int32_t *e_off;           // [E + 1]
    int32_t *e_tok;           // [2T]
    int32_t *pos;             // [T x 2] list position of (token, k)
    const float *Ypart;       // [kSplitK x 2T x d]
    int rows_cap;
};

constexpr int kNormThreads = 256;
constexpr int kMaxD = 8192;
__global__ void __launch_bounds__(kNormThreads) k_norm_route(TokenParams p)
{
    const int t = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const float *r = p.resid + size_t(t) * p.d;
    __shared__ float red[32];
    __shared__ float lg[kMaxExperts];
    __shared__ float xs[kMaxD];
    // sum of squares (vectorised, fixed order: threads, then warps)
    float ss = 0.f;
    for (int j = 4 * tid; j < p.d; j += 4 * kNormThreads) {
        const float4 v = *reinterpret_cast<const float4 *>(r + j);
        *reinterpret_cast<float4 *>(xs + j) = v;
        ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
    }
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    if (tid == 0) {
        float a = 0.f;
        for (int w = 0; w < kNormThreads / 32; ++w) a += red[w];
        red[31] = 1.f / sqrtf(a / float(p.d) + p.eps);
    }
    __syncthreads();
    const float inv = red[31];
    for (int j = tid; j < p.d; j += kNormThreads) {
        const float x = xs[j] * inv;
        xs[j] = x;
        if (p.x_bf16) reinterpret_cast<__nv_bfloat16 *>(p.X16)[size_t(t) * p.d + j] = __float2bfloat16_rn(x);
        else reinterpret_cast<__half *>(p.X16)[size_t(t) * p.d + j] = __float2half_rn(x);
    }
    if (p.E > 1) {
        __syncthreads();
        // router logits in fp32: warp w takes experts w, w + 8, ...; lanes run
        // over 8-element pieces of the router row
        for (int e = warp; e < p.E; e += kNormThreads / 32) {
            const __half *row = p.router + size_t(e) * p.d;
            float a = 0.f;
            for (int j = 8 * lane; j < p.d; j += 8 * 32) {
                const uint4 q = *reinterpret_cast<const uint4 *>(row + j);
                const __half2 *h2 = reinterpret_cast<const __half2 *>(&q);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f = __half22float2(h2[i]);
                    a = fmaf(f.x, xs[j + 2 * i], fmaf(f.y, xs[j + 2 * i + 1], a));
                }
            }
            for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
            if (lane == 0) lg[e] = a;
        }
        __syncthreads();
        if (tid == 0) {
            float mx = -INFINITY, pr[kMaxExperts], den = 0.f;
            for (int e = 0; e < p.E; ++e) mx = fmaxf(mx, lg[e]);
            for (int e = 0; e < p.E; ++e) { pr[e] = expf(lg[e] - mx); den += pr[e]; }
            for (int e = 0; e < p.E; ++e) pr[e] /= den;
            int ea = 0;
            for (int e = 1; e < p.E; ++e) if (pr[e] > pr[ea]) ea = e;
            int eb = ea == 0 ? 1 : 0;
            for (int e = 0; e < p.E; ++e) if (e != ea && pr[e] > pr[eb]) eb = e;
            const int lo = min(ea, eb), hi = max(ea, eb);
            p.route_e[2 * t] = lo;
            p.route_e[2 * t + 1] = hi;
            p.route_w[2 * t] = pr[lo] / (pr[lo] + pr[hi]);
            p.route_w[2 * t + 1] = pr[hi] / (pr[lo] + pr[hi]);
        }
    } else if (tid == 0) {
        p.route_e[2 * t] = 0;
        p.route_e[2 * t + 1] = -1;
        p.route_w[2 * t] = 1.f;
        p.route_w[2 * t + 1] = 0.f;
    }
}

// Counting sort of the (token, slot) items by expert, items taken in
// ascending (token, slot) order so each expert's list is in ascending token
// order: deterministic.  One CTA of 1024 threads; per chunk of 1024 items,
// warp ballots give each item its rank among the chunk's items of the same
// expert before it.
constexpr int kSortThreads = 1024;
__global__ void __launch_bounds__(kSortThreads) k_sort(TokenParams p)
{
    __shared__ int tot[kMaxExperts];
    __shared__ int base[kMaxExperts];
    __shared__ int wcnt[kSortThreads / 32][kMaxExperts];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = p.T * p.top_k;
    if (tid < kMaxExperts) tot[tid] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += kSortThreads) atomicAdd(&tot[p.route_e[2 * (i / p.top_k) + i % p.top_k]], 1);
    __syncthreads();
    if (tid == 0) {
        int acc = 0;
        for (int e = 0; e < p.E; ++e) {
            p.e_off[e] = acc;
            base[e] = acc;
            acc += tot[e];
        }
        p.e_off[p.E] = acc;
    }
    __syncthreads();
    const unsigned lt = (1u << lane) - 1u;
    for (int c0 = 0; c0 < n; c0 += kSortThreads) {
        const int i = c0 + tid;
        const int t = i / p.top_k, k = i % p.top_k;
        const int e = i < n ? p.route_e[2 * t + k] : -1;
        int rank = 0;
        for (int x = 0; x < p.E; ++x) {
            const unsigned m = __ballot_sync(0xffffffffu, e == x);
            if (e == x) rank = __popc(m & lt);
            if (lane == 0) wcnt[warp][x] = __popc(m);
        }
        __syncthreads();
        if (e >= 0) {
            int q = base[e] + rank;
            for (int w = 0; w < warp; ++w) q += wcnt[w][e];
            p.e_tok[q] = t;
            p.pos[2 * t + k] = q;
        }
        __syncthreads();
        if (tid < p.E) {
            int s = 0;
            for (int w = 0; w < kSortThreads / 32; ++w) s += wcnt[w][tid];
            base[tid] += s;
        }
        __syncthreads();
    }
}

// The normalised inputs in list order (rows of each expert's tokens
// contiguous), for the tensor-map loads of the gate/up GEMM.  16-bit elements.
__global__ void k_gather_x(TokenParams p, uint8_t *__restrict__ xs)
{
    const int q = blockIdx.x;
    if (q >= p.e_off[p.E]) return;
    const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(p.X16) + size_t(p.e_tok[q]) * p.d * 2);
    uint4 *dst = reinterpret_cast<uint4 *>(xs + size_t(q) * p.d * 2);
    for (int i = threadIdx.x; i < p.d / 8; i += blockDim.x) dst[i] = src[i];
}

// r += sum over the token's experts (ascending index) of w * (sum of the
// K-split partials in split order)
__global__ void k_combine(TokenParams p)
{
    const int t = blockIdx.x;
    for (int j = 4 * threadIdx.x; j < p.d; j += 4 * blockDim.x) {
        float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int k = 0; k < p.top_k; ++k) {
            const int q = p.pos[2 * t + k];
            float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int sp = 0; sp < kSplitK; ++sp) {
                const float4 v = *reinterpret_cast<const float4 *>(p.Ypart + (size_t(sp) * p.rows_cap + q) * p.d + j);
                a.x += v.x; a.y += v.y; a.z += v.z; a.w += v.w;
            }
            const float w = p.route_w[2 * t + k];
            y.x = fmaf(w, a.x, y.x); y.y = fmaf(w, a.y, y.y); y.z = fmaf(w, a.z, y.z); y.w = fmaf(w, a.w, y.w);
        }
        float4 *rr = reinterpret_cast<float4 *>(p.resid + size_t(t) * p.d + j);
        float4 r = *rr;
        r.x += y.x; r.y += y.y; r.z += y.z; r.w += y.w;
        *rr = r;
    }
}

}  // namespace

// ---------------------------------------------------------------------------
// Host
// ---------------------------------------------------------------------------
// The tensor-map encoder is a driver entry point, looked up through the
// runtime so that the library has no link-time dependency on the driver.
typedef CUresult (*TensorMapEncodeFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                      const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                      CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                      CUtensorMapFloatOOBfill);
static TensorMapEncodeFn tensor_map_encoder()
{
    static TensorMapEncodeFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<TensorMapEncodeFn>(ptr);
    }
    return fn;
}
struct PrefillState {
    int T = 0, d = 0, F = 0;
    uint8_t *buf = nullptr;
    size_t bytes = 0;
    // INT4 weight tensor maps per layer and expert: gate/up nibbles, gate/up
    // scales, down nibbles, down scales (encoded on first use, dropped when the
    // layer is reloaded)
    std::vector<CUtensorMap> wmaps;
    std::vector<char> wmaps_ok;
};

static size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

int prefill_run(PrefillState **state, const PrefillView &v, int l0, int l1, int T, float *resid,
                cudaStream_t stream, char *msg, int msg_len)
{
    if (v.wfmt != kF16 && v.wfmt != kBF16 && v.wfmt != kI4) {
        snprintf(msg, msg_len, "dense prefill supports F16, BF16 and INT4G32 weights");
        return 1;
    }
    if (v.d % BN != 0 || v.F % (BN / 2) != 0 || v.F % BK != 0 || v.d % BK != 0) {
        snprintf(msg, msg_len, "dense prefill needs d_model %% 256 == 0 and d_ff %% 128 == 0");
        return 1;
    }
    const int rows_cap = 2 * T;
    const size_t o_x16 = 0;
    const size_t o_xs = up256(o_x16 + sizeof(__half) * size_t(T) * v.d);
    const size_t o_h = up256(o_xs + sizeof(__half) * size_t(rows_cap) * v.d);
    const size_t o_y = up256(o_h + sizeof(__half) * size_t(rows_cap) * v.F);
    const size_t o_re = up256(o_y + sizeof(float) * size_t(kSplitK) * rows_cap * v.d);
    const size_t o_rw = up256(o_re + sizeof(int32_t) * 2 * T);
    const size_t o_eo = up256(o_rw + sizeof(float) * 2 * T);
    const size_t o_et = up256(o_eo + sizeof(int32_t) * (kMaxExperts + 1));
    const size_t o_pos = up256(o_et + sizeof(int32_t) * rows_cap);
    const size_t total = up256(o_pos + sizeof(int32_t) * 2 * T);
    PrefillState *st = *state;
    if (!st || st->bytes < total) {
        if (st) cudaFree(st->buf);
        if (!st) st = new PrefillState;
        *state = st;
        st->buf = nullptr;
        st->bytes = 0;
        if (cudaMalloc(&st->buf, total) != cudaSuccess) {
            snprintf(msg, msg_len, "prefill workspace allocation of %zu bytes failed", total);
            return 3;
        }
        st->bytes = total;
    }
    uint8_t *B = st->buf;
    // element type of the MMA operands: 0 f16, 1 bf16, 2 INT4 dequantised to f16
    const int W = v.wfmt == kBF16 ? 1 : (v.wfmt == kI4 ? 2 : 0);
    void (*gu)(GemmParams) = W == 0 ? k_gemm<kGU, 0> : (W == 1 ? k_gemm<kGU, 1> : k_gemm<kGU, 2>);
    void (*dn)(GemmParams) = W == 0 ? k_gemm<kDOWN, 0> : (W == 1 ? k_gemm<kDOWN, 1> : k_gemm<kDOWN, 2>);
    // per device and kernel; cheap enough to repeat per call
    const int smem_bytes = W == 2 ? kGemmSmemI4 : kGemmSmem;
    if (cudaFuncSetAttribute(gu, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) != cudaSuccess ||
        cudaFuncSetAttribute(dn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) != cudaSuccess) {
        snprintf(msg, msg_len, "prefill: cudaFuncSetAttribute: %s", cudaGetErrorString(cudaGetLastError()));
        return 2;
    }

    TokenParams tp{};
    tp.resid = resid;
    tp.X16 = B + o_x16;
    tp.x_bf16 = W == 1;
    tp.d = v.d;
    tp.E = v.E;
    tp.T = T;
    tp.top_k = v.top_k;
    tp.eps = v.eps;
    tp.route_e = reinterpret_cast<int32_t *>(B + o_re);
    tp.route_w = reinterpret_cast<float *>(B + o_rw);
    tp.e_off = reinterpret_cast<int32_t *>(B + o_eo);
    tp.e_tok = reinterpret_cast<int32_t *>(B + o_et);
    tp.pos = reinterpret_cast<int32_t *>(B + o_pos);
    tp.Ypart = reinterpret_cast<const float *>(B + o_y);
    tp.rows_cap = rows_cap;

    GemmParams gp{};
    gp.E = v.E;
    gp.d = v.d;
    gp.F = v.F;
    gp.gated = v.gated;
    gp.act = v.act;
    gp.wrow = v.wrow;
    gp.rec_bytes = v.rec_bytes;
    gp.wd_stride = v.wd_stride;
    gp.e_off = tp.e_off;
    gp.e_tok = tp.e_tok;
    gp.H = B + o_h;
    gp.Ypart = reinterpret_cast<float *>(B + o_y);
    gp.rows_cap = rows_cap;
    gp.err = v.err;
    gp.wait_ns = v.wait_ns;
    gp.debug_flags = v.debug_flags;
    const int mtiles = (rows_cap + kTileRows - 1) / kTileRows + v.E;   // upper bound over experts
    // tensor maps of the A operands: rows_cap rows of K 16-bit elements,
    // boxes of 64 elements (128 bytes) x 128 rows, 128-byte swizzle
    CUtensorMap tm_gu, tm_dn;
    {
        const CUtensorMapDataType dt = W == 1 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
        const TensorMapEncodeFn enc = tensor_map_encoder();
        if (!enc) {
            snprintf(msg, msg_len, "prefill: the driver offers no cuTensorMapEncodeTiled");
            return 2;
        }
        auto encode = [&](CUtensorMap *m, void *base, int K) -> CUresult {
            const cuuint64_t gdim[2] = {cuuint64_t(K), cuuint64_t(rows_cap)};
            const cuuint64_t gstride[1] = {cuuint64_t(K) * 2};
            const cuuint32_t box[2] = {BK, BM};
            const cuuint32_t estr[2] = {1, 1};
            return enc(m, dt, 2, base, gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        };
        if (encode(&tm_gu, B + o_xs, v.d) != CUDA_SUCCESS || encode(&tm_dn, B + o_h, v.F) != CUDA_SUCCESS) {
            snprintf(msg, msg_len, "prefill: cuTensorMapEncodeTiled failed");
            return 2;
        }
    }

    if (W == 2) {
        // INT4 weights as bytes: gate/up rows {wrow bytes} x {gate, up} x F
        // neurons (rec_bytes apart), down rows {wrow bytes} x F (wd_stride apart)
        const TensorMapEncodeFn enc = tensor_map_encoder();
        const size_t nl = v.n_layers;
        if (st->wmaps.size() != nl * v.E * 4) {
            st->wmaps.assign(nl * v.E * 4, CUtensorMap{});
            st->wmaps_ok.assign(nl, 0);
        }
        const int G = v.gated ? 2 : 1;
        for (int l = l0; l < l1; ++l) {
            if (st->wmaps_ok[l]) continue;
            for (int e = 0; e < v.E; ++e) {
                const ExpertDev &x = v.ex[size_t(l) * v.E + e];
                CUtensorMap *m = &st->wmaps[(size_t(l) * v.E + e) * 4];
                const cuuint64_t gdim3[3] = {cuuint64_t(v.wrow), cuuint64_t(G), cuuint64_t(v.F)};
                const cuuint64_t gstr3[2] = {cuuint64_t(v.wrow), cuuint64_t(v.rec_bytes)};
                const cuuint32_t boxw[3] = {BK / 2, cuuint32_t(G), BN / 2}, boxs[3] = {16, cuuint32_t(G), BN / 2};
                const cuuint32_t es3[3] = {1, 1, 1};
                const cuuint64_t gdim2[2] = {cuuint64_t(v.wrow), cuuint64_t(v.F)};
                const cuuint64_t gstr2[1] = {cuuint64_t(v.wd_stride)};
                const cuuint32_t boxdw[2] = {128, BK}, boxds[2] = {16, BK};
                const cuuint32_t es2[2] = {1, 1};
                const CUtensorMapDataType u8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
                if (enc(&m[0], u8, 3, const_cast<uint8_t *>(x.Wgu), gdim3, gstr3, boxw, es3,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
                    enc(&m[1], u8, 3, const_cast<uint8_t *>(x.Wgu), gdim3, gstr3, boxs, es3,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
                    enc(&m[2], u8, 2, const_cast<uint8_t *>(x.Wd), gdim2, gstr2, boxdw, es2,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
                    enc(&m[3], u8, 2, const_cast<uint8_t *>(x.Wd), gdim2, gstr2, boxds, es2,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
                    snprintf(msg, msg_len, "prefill: cuTensorMapEncodeTiled failed for the INT4 weights");
                    return 2;
                }
            }
            st->wmaps_ok[l] = 1;
        }
    }

    for (int l = l0; l < l1; ++l) {
        tp.router = v.E > 1 ? reinterpret_cast<const __half *>(v.router[l]) : nullptr;
        for (int e = 0; e < v.E; ++e) {
            const ExpertDev &x = v.ex[size_t(l) * v.E + e];
            gp.ex[e] = PrefillExpert{x.Wgu, x.Wd, x.c};
        }
        k_norm_route<<<T, kNormThreads, 0, stream>>>(tp);
        k_sort<<<1, kSortThreads, 0, stream>>>(tp);
        k_gather_x<<<rows_cap, 128, 0, stream>>>(tp, B + o_xs);
        dim3 g1(2 * v.F / BN, mtiles, 1);
        gp.tmA = tm_gu;
        if (W == 2)
            for (int e = 0; e < v.E; ++e) {
                gp.tmW[e] = st->wmaps[(size_t(l) * v.E + e) * 4 + 0];
                gp.tmS[e] = st->wmaps[(size_t(l) * v.E + e) * 4 + 1];
            }
        gu<<<g1, kGemmThreads, smem_bytes, stream>>>(gp);
        dim3 g2(v.d / BN, mtiles, kSplitK);
        gp.tmA = tm_dn;
        if (W == 2)
            for (int e = 0; e < v.E; ++e) {
                gp.tmW[e] = st->wmaps[(size_t(l) * v.E + e) * 4 + 2];
                gp.tmS[e] = st->wmaps[(size_t(l) * v.E + e) * 4 + 3];
            }
        dn<<<g2, kGemmThreads, smem_bytes, stream>>>(gp);
        k_combine<<<T, 256, 0, stream>>>(tp);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) {
            snprintf(msg, msg_len, "prefill launch: %s", cudaGetErrorString(e));
            return 2;
        }
    }
    return 0;
}

void prefill_invalidate(PrefillState *st, int layer)
{
    if (st && layer >= 0 && layer < int(st->wmaps_ok.size())) st->wmaps_ok[layer] = 0;
}

void prefill_destroy(PrefillState *state)
{
    if (!state) return;
    cudaFree(state->buf);
    delete state;
}

}  // namespace pi
