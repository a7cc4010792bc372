// pi_decode.cu -- persistent sparse-FFN decode kernel for sm_100a.
//
// One cooperative launch runs a range of layers for one token.  Each CTA owns
// one strip of the neuron table (a contiguous run of table positions holding
// a balanced share of hot neurons, hottest first) and a slice of the rows of
// t = V x.  Per layer:
//
//   phase A  x = RMSNorm(r) (every CTA, identical arithmetic); [MoE] router +
//            top-2 (every CTA, identical); the CTA's rows of t = V x.
//   --- grid barrier ---
//   phase B  z = U t - c over the strip; active iff z > threshold; the active
//            list is compacted in ascending table order with warp ballots
//            (PowerInfer (unite.ai), "Adaptive sparse predictor").
//   phase C  for active neurons only: the neuron's W_gate / W_up rows ->
//            h = act(g, u); for h != 0 its W_down column (stored as a row) is
//            accumulated into a per-CTA fp32 partial of y ("Neuron-aware
//            operators": rows of the input matrices, columns of the output).
//   --- grid barrier ---
//   phase D  r <- r + sum of the per-CTA partials in fixed CTA order, by
//            column slices (deterministic, no atomics): the merge of partial
//            results (nearauto.com PowerInfer article, Fig. 8).
//   --- grid barrier ---
//
// Memory strategy: every weight byte is first pulled into L2 with
// cp.async.bulk.prefetch.L2 as early as its address is known -- the next
// layer's predictor slice (V rows, U strip) while the current layer gathers,
// a strip's active neuron records the moment its active list exists (and,
// for ReLU / ReGLU, where h != 0 almost always follows z > 0, their W_down
// rows too) -- and the 16 warps then read it with batched 128-bit loads:
// many rows in flight per thread and one cross-warp reduction per batch.
// The gather is software-pipelined: the W_down rows of batch i and the
// W_gate/W_up records of batch i+1 are loaded together.  HBM traffic is the
// algorithmic bytes (plus the speculative W_down rows whose h turns out 0).
// All waits are bounded (%globaltimer); a wait that runs out records an
// error word and every thread of the grid returns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

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
// Stored formats.  A vector is 16 bytes of a row (8 bytes for INT4: 16
// nibbles, half of a 32-element scale group).
// ---------------------------------------------------------------------------
template <int F> struct Fm;
template <> struct Fm<kF32>  { static constexpr int VB = 16, EPV = 4;  using V = uint4; };
template <> struct Fm<kF16>  { static constexpr int VB = 16, EPV = 8;  using V = uint4; };
template <> struct Fm<kBF16> { static constexpr int VB = 16, EPV = 8;  using V = uint4; };
template <> struct Fm<kI4>   { static constexpr int VB = 8,  EPV = 16; using V = uint2; };

template <int F>
__device__ __forceinline__ typename Fm<F>::V ldvec(const uint8_t *p)
{
    if constexpr (F == kI4) return ldw2(p);
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
    } else {
        // element 2j sits in the low nibble of byte j; n - 8 is formed exactly
        // by placing n in the mantissa of 2^23 and subtracting 2^23 + 8
        const uint32_t w[2] = {v.x, v.y};
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j)
                o[8 * i + j] = __uint_as_float(0x4b000000u | ((w[i] >> (4 * j)) & 0xfu)) - 8388616.0f;
    }
}

// Scale of the 32-element group holding INT4 vector v of a row record
// (d/2 nibble bytes, then one fp16 scale per 32 elements).
__device__ __forceinline__ float i4_scale(const uint8_t *row, int d, int v)
{
    const unsigned short s = __ldg(reinterpret_cast<const unsigned short *>(row + d / 2) + (v >> 1));
    return __half2float(__ushort_as_half(s));
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float act_h(int act, float g, float u)
{
    const float gp = g > 0.f ? g : 0.f;
    if (act == 0) return gp;               // ReLU (non-gated)
    if (act == 1) return gp * u;           // ReGLU
    return gp * (u > 0.f ? u : 0.f);       // dReLU
}

constexpr int kNB = 4;            // neurons per gather batch
constexpr int kRA = 16;           // V rows per staging round at most
constexpr int kMaxU = 4;          // U vectors per lane (rank <= 128 * EPV)
constexpr int kRed = 2 * kNB > kRA ? 2 * kNB : kRA;

struct Smem {
    float red[2][kConsumerWarps][kRed];
    alignas(16) float tsm[kMaxRankTotal];
    float cbuf[kMaxTopK][kMaxStrip];
    float zbuf[kMaxTopK][kMaxStrip];
    int16_t lst[kMaxTopK * kMaxStrip];     // active neurons: (slot << 12) | local
    int lst_n[kMaxTopK];
    int16_t nz[kMaxTopK * kMaxStrip];      // neurons with h != 0, same encoding
    float hz[kMaxTopK * kMaxStrip];        // their h (routing weight folded in)
    int nz_n;
    int route_e[kMaxTopK];
    float route_w[kMaxTopK];
    float lg[kConsumerWarps][kMaxExperts];
    float inv_rms;
    int bc[2];
    uint64_t stage_bar;                    // completion of a staging round
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

// Grid-wide barrier of all CTAs of the cooperative launch: arrivals are
// fire-and-forget releases on one counter (never reset within a launch);
// thread 0 of each CTA polls it with acquire loads, bounded by wait_ns.  The
// outcome is broadcast through shared memory so the whole CTA agrees.
__device__ bool grid_sync(Smem *sm, const DecodeParams &p, unsigned &epoch, int &bci, long long *cyc)
{
    cta_sync();
    if (threadIdx.x == 0) {
        const long long c0 = clock64();
        bool ok = true;
        epoch += 1;
        unsigned target = epoch * gridDim.x;
        if ((p.debug_flags & 1) && epoch == 1) target += 1;   // PI_DEBUG_STALL_BARRIER
        __threadfence();
        red_release_gpu(p.bar, 1u);
        const long long t0 = gtimer();
        unsigned it = 0;
        while (ld_acquire_gpu(p.bar) < target) {
            if ((++it & 31) == 0 && gtimer() - t0 > p.wait_ns) {
                set_error(p.err, kDevTimeout);
                ok = false;
                break;
            }
        }
        __threadfence();
        st_vol(&sm->bc[bci], ok ? 1 : 0);
        if (cyc) *cyc += clock64() - c0;
    }
    cta_sync();
    const bool ok = ld_vol(&sm->bc[bci]) != 0;
    bci ^= 1;
    return ok;
}

// Staging round: thread 0 has issued bulk copies of `bytes` in total onto
// sm->stage_bar; it waits (bounded) and the whole CTA adopts its verdict.
__device__ bool stage_wait(Smem *sm, const DecodeParams &p, uint32_t &par, int &bci)
{
    if (threadIdx.x == 0) {
        bool ok = mbar_test(&sm->stage_bar, par);
        if (!ok) {
            const long long t0 = gtimer();
            for (unsigned it = 1; !ok; ++it) {
                ok = mbar_test(&sm->stage_bar, par);
                if (!ok && (it & 15) == 0 && gtimer() - t0 > p.wait_ns) {
                    set_error(p.err, kDevTimeout);
                    break;
                }
            }
        }
        st_vol(&sm->bc[bci], ok ? 1 : 0);
    }
    cta_sync();
    const bool ok = ld_vol(&sm->bc[bci]) != 0;
    bci ^= 1;
    if (ok) mbar_test(&sm->stage_bar, par);   // acquire for this thread (phase complete)
    par ^= 1;
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
template <int WF, int PF, int DMAX>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ DecodeParams p)
{
    constexpr int EPVW = Fm<WF>::EPV, EPVP = Fm<PF>::EPV, VBW = Fm<WF>::VB, VBP = Fm<PF>::VB;
    constexpr int MAXVW = (DMAX / EPVW + kThreads - 1) / kThreads;
    constexpr int MAXVP = (DMAX / EPVP + kThreads - 1) / kThreads;
    // neurons per gather batch: fewer when a row takes several vectors per thread
    constexpr int NB = MAXVW >= 2 ? kNB / 2 : kNB;
    // when both formats share the vector layout, x is cached once
    constexpr bool kSameX = (WF == PF);
    using VW = typename Fm<WF>::V;
    using VP = typename Fm<PF>::V;

    __shared__ Smem sm;
    extern __shared__ __align__(128) uint8_t stg[];   // kStageBytes staging buffer
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.x, S = gridDim.x;
    const int d = p.d, r = p.r;
    const int s0 = p.strip_off[b], ns = p.strip_off[b + 1] - s0;
    const bool predict = p.mode == kModePredict;
    const int ntop = predict ? 1 : p.top_k;
    const int rows_total = ntop * r;
    const int a0 = int((long long)b * rows_total / S), a1 = int((long long)(b + 1) * rows_total / S);
    const int nvecW = (WF == kI4 ? d / 2 : d * (WF == kF32 ? 4 : 2)) / VBW;
    const int nvecP = p.vrow / VBP;
    const int nvecU = p.urow / VBP;
    const int l0 = p.layer_begin;
    const int l1 = predict ? p.layer_begin + 1 : p.layer_end;
    const bool dense_ahead = !predict && p.E == 1;

    // L2 prefetch of a layer's predictor slice of this CTA: V rows [a0, a1)
    // of the concatenated experts and the U strip of each expert.
    auto prefetch_pred = [&](int l, const int *experts, bool want_v, bool want_u) {
        for (int e = 0; e < ntop; ++e) {
            const ExpertDev &ex = p.ex[size_t(l) * p.E + experts[e]];
            const int lo = max(a0, e * r), hi = min(a1, (e + 1) * r);
            if (want_v && hi > lo)
                prefetch_l2(ex.V + size_t(lo - e * r) * p.vrow, uint32_t(hi - lo) * p.vrow);
            if (want_u && ns > 0)
                prefetch_l2(ex.U + size_t(s0) * p.urow, uint32_t(ns) * p.urow);
        }
    };

    if (tid == 0) {
        mbar_init(&sm.stage_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        if (predict) {
            const int ex[kMaxTopK] = {p.pred_expert, 0};
            prefetch_pred(l0, ex, true, true);
        } else if (dense_ahead) {
            const int ex[kMaxTopK] = {0, 0};
            prefetch_pred(l0, ex, true, true);
        }
    }

    cta_sync();
    unsigned epoch = 0;
    uint32_t spar = 0;
    int bci = 0;
    float xw[MAXVW * EPVW];
    float xp_own[kSameX ? 1 : MAXVP * EPVP];
#define XP(i) (kSameX ? xw[(i)] : xp_own[(i)])
    int rb = 0;

    for (int l = l0; l < l1; ++l) {
        const int li = l - l0;
        long long cyc_a = 0, cyc_b = 0, cyc_c = 0, cyc_bar = 0;
        prof_put(p, li, 0, gtimer());
        const long long ca0 = clock64();

        // ---------------- phase A: layer input ------------------------------
        const float *src = predict ? p.x_in : p.resid;
#pragma unroll
        for (int k = 0; k < MAXVW; ++k) {
            const int v = tid + kThreads * k;
#pragma unroll
            for (int i = 0; i < EPVW; i += 4) {
                float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
                if (v < nvecW) q = __ldcg(reinterpret_cast<const float4 *>(src + v * EPVW + i));
                xw[k * EPVW + i] = q.x; xw[k * EPVW + i + 1] = q.y;
                xw[k * EPVW + i + 2] = q.z; xw[k * EPVW + i + 3] = q.w;
            }
        }
        if constexpr (!kSameX) {
#pragma unroll
            for (int k = 0; k < MAXVP; ++k) {
                const int v = tid + kThreads * k;
#pragma unroll
                for (int i = 0; i < EPVP; i += 4) {
                    float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (v < nvecP) q = __ldcg(reinterpret_cast<const float4 *>(src + v * EPVP + i));
                    xp_own[k * EPVP + i] = q.x; xp_own[k * EPVP + i + 1] = q.y;
                    xp_own[k * EPVP + i + 2] = q.z; xp_own[k * EPVP + i + 3] = q.w;
                }
            }
        }
        if (!predict) {
            // x = r / sqrt(mean(r^2) + eps); the W-format columns cover d once
            float ss = 0.f;
#pragma unroll
            for (int k = 0; k < MAXVW; ++k) {
                const int v = tid + kThreads * k;
                if (v < nvecW) {
#pragma unroll
                    for (int i = 0; i < EPVW; ++i) ss = fmaf(xw[k * EPVW + i], xw[k * EPVW + i], ss);
                    if (p.trace && b == 0) {
#pragma unroll
                        for (int i = 0; i < EPVW; i += 4)
                            __stcg(reinterpret_cast<float4 *>(p.trace + size_t(li) * d + v * EPVW + i),
                                   make_float4(xw[k * EPVW + i], xw[k * EPVW + i + 1],
                                               xw[k * EPVW + i + 2], xw[k * EPVW + i + 3]));
                    }
                }
            }
            ss = warp_sum(ss);
            if (lane == 0) sm.red[rb][warp][0] = ss;
            cta_sync();
            if (tid == 0) {
                float tot = 0.f;
                for (int w = 0; w < kConsumerWarps; ++w) tot += sm.red[rb][w][0];
                sm.inv_rms = 1.f / sqrtf(tot / float(d) + p.eps);
            }
            cta_sync();
            rb ^= 1;
            const float inv = sm.inv_rms;
#pragma unroll
            for (int i = 0; i < MAXVW * EPVW; ++i) xw[i] *= inv;
            if constexpr (!kSameX) {
#pragma unroll
                for (int i = 0; i < MAXVP * EPVP; ++i) xp_own[i] *= inv;
            }
        }
        prof_put(p, li, 1, gtimer());

        // MoE routing, computed identically by every CTA: logits of the E
        // experts (fp16 router, 8-element vectors like the predictor format),
        // softmax, two largest (ties: lower index), weights renormalised over
        // the two, experts in ascending index.
        if (!predict && p.E > 1) {
            const uint8_t *R = p.router[l];
            float lg[kMaxExperts];
#pragma unroll
            for (int e = 0; e < kMaxExperts; ++e) {
                lg[e] = 0.f;
                if (e < p.E) {
#pragma unroll
                    for (int k = 0; k < MAXVP; ++k) {
                        const int v = tid + kThreads * k;
                        if (v < nvecP) {
                            float w[8];
                            cvt<kF16>(ldw4(R + (size_t(e) * nvecP + v) * 16), w);
#pragma unroll
                            for (int i = 0; i < 8; ++i) lg[e] = fmaf(w[i], XP(k * EPVP + i), lg[e]);
                        }
                    }
                }
            }
#pragma unroll
            for (int e = 0; e < kMaxExperts; ++e) {
                if (e < p.E) {
                    const float v = warp_sum(lg[e]);
                    if (lane == 0) sm.lg[warp][e] = v;
                }
            }
            cta_sync();
            if (tid == 0) {
                float logit[kMaxExperts];
                float mx = -INFINITY;
                for (int e = 0; e < p.E; ++e) {
                    float s = 0.f;
                    for (int w = 0; w < kConsumerWarps; ++w) s += sm.lg[w][e];
                    logit[e] = s;
                    mx = fmaxf(mx, s);
                }
                float pr[kMaxExperts];
                float den = 0.f;
                for (int e = 0; e < p.E; ++e) { pr[e] = expf(logit[e] - mx); den += pr[e]; }
                for (int e = 0; e < p.E; ++e) pr[e] /= den;
                int ea = 0;
                for (int e = 1; e < p.E; ++e) if (pr[e] > pr[ea]) ea = e;
                int eb = ea == 0 ? 1 : 0;
                for (int e = 0; e < p.E; ++e) if (e != ea && pr[e] > pr[eb]) eb = e;
                const int lo = min(ea, eb), hi = max(ea, eb);
                sm.route_e[0] = lo;
                sm.route_e[1] = hi;
                sm.route_w[0] = pr[lo] / (pr[lo] + pr[hi]);
                sm.route_w[1] = pr[hi] / (pr[lo] + pr[hi]);
                if (p.stats && b == 0) {
                    p.stats[li * 4 + 2] = lo;
                    p.stats[li * 4 + 3] = hi;
                }
                // the two experts' predictor slices start moving now
                prefetch_pred(l, sm.route_e, true, true);
            }
        } else if (tid == 0) {
            sm.route_e[0] = predict ? p.pred_expert : 0;
            sm.route_e[1] = 0;
            sm.route_w[0] = 1.f;
            sm.route_w[1] = 0.f;
            if (p.stats && b == 0 && !predict) {
                p.stats[li * 4 + 2] = -1;
                p.stats[li * 4 + 3] = -1;
            }
        }
        cta_sync();

        // ---------------- phase A: t rows [a0, a1) ---------------------------
        // staged through shared memory in rounds of up to kRA rows
        {
            const int per = min(kRA, kStageBytes / p.vrow);
            bool ok = true;
            for (int row0 = a0; row0 < a1 && ok; row0 += per) {
                const int n = min(per, a1 - row0);
                if (tid == 0) {
                    mbar_arrive_tx(&sm.stage_bar, uint32_t(n) * p.vrow);
                    // the rows of one round lie in at most two experts' V
                    for (int rr = 0; rr < n;) {
                        const int row = row0 + rr, e = row / r;
                        const int cnt = min(n - rr, (e + 1) * r - row);
                        const uint8_t *vrow =
                            p.ex[size_t(l) * p.E + sm.route_e[e]].V + size_t(row - e * r) * p.vrow;
                        stage_copy(stg + size_t(rr) * p.vrow, vrow, uint32_t(cnt) * p.vrow, &sm.stage_bar);
                        rr += cnt;
                    }
                }
                if (!stage_wait(&sm, p, spar, bci)) { ok = false; break; }
                float part[kRA];
#pragma unroll
                for (int rr = 0; rr < kRA; ++rr) {
                    part[rr] = 0.f;
                    if (rr < n) {
#pragma unroll
                        for (int k = 0; k < MAXVP; ++k) {
                            const int v = tid + kThreads * k;
                            if (v < nvecP) {
                                float w[EPVP];
                                cvt<PF>(*reinterpret_cast<const VP *>(stg + size_t(rr) * p.vrow + v * VBP), w);
#pragma unroll
                                for (int i = 0; i < EPVP; ++i) part[rr] = fmaf(w[i], XP(k * EPVP + i), part[rr]);
                            }
                        }
                    }
                }
#pragma unroll
                for (int rr = 0; rr < kRA; ++rr) {
                    if (rr < n) {
                        const float v = warp_sum(part[rr]);
                        if (lane == 0) sm.red[rb][warp][rr] = v;
                    }
                }
                cta_sync();
                if (tid < n) {
                    float t = 0.f;
                    for (int w = 0; w < kConsumerWarps; ++w) t += sm.red[rb][w][tid];
                    __stcg(p.t_buf + row0 + tid, t);
                }
                rb ^= 1;
            }
            if (!ok) break;
        }
        cyc_a = clock64() - ca0;
        prof_put(p, li, 2, gtimer());
        if (!grid_sync(&sm, p, epoch, bci, &cyc_bar)) break;
        prof_put(p, li, 3, gtimer());

        // ---------------- phase B: z = U t - c, threshold, compaction --------
        const long long cb0 = clock64();
        {
            constexpr int kTV = kMaxRankTotal / kThreads;
            float tv[kTV];
#pragma unroll
            for (int k = 0; k < kTV; ++k) {
                const int i = tid + kThreads * k;
                tv[k] = i < ntop * r ? __ldcg(p.t_buf + i) : 0.f;
            }
            float cv[kMaxTopK];
#pragma unroll
            for (int e = 0; e < kMaxTopK; ++e)
                cv[e] = (e < ntop && tid < ns) ? __ldg(p.ex[size_t(l) * p.E + sm.route_e[e]].c + s0 + tid)
                                               : 0.f;
#pragma unroll
            for (int k = 0; k < kTV; ++k) {
                const int i = tid + kThreads * k;
                if (i < ntop * r) sm.tsm[i] = tv[k];
            }
#pragma unroll
            for (int e = 0; e < kMaxTopK; ++e)
                if (e < ntop && tid < ns) sm.cbuf[e][tid] = cv[e];
        }
        cta_sync();
        {
            bool ok = true;
            const int per = kStageBytes / p.urow;   // U rows per staging round
            for (int e = 0; e < ntop && ok; ++e) {
                const float *te = sm.tsm + e * r;
                const uint8_t *U = p.ex[size_t(l) * p.E + sm.route_e[e]].U + size_t(s0) * p.urow;
                for (int row0 = 0; row0 < ns && ok; row0 += per) {
                    const int n = min(per, ns - row0);
                    if (tid == 0) {
                        mbar_arrive_tx(&sm.stage_bar, uint32_t(n) * p.urow);
                        stage_copy(stg, U + size_t(row0) * p.urow, uint32_t(n) * p.urow, &sm.stage_bar);
                    }
                    if (!stage_wait(&sm, p, spar, bci)) { ok = false; break; }
                    for (int rr = warp; rr < n; rr += kConsumerWarps) {
                        const uint8_t *urow = stg + size_t(rr) * p.urow;
                        float a = 0.f;
#pragma unroll
                        for (int k = 0; k < kMaxU; ++k) {
                            const int v = lane + 32 * k;
                            if (v < nvecU) {
                                float w[EPVP];
                                cvt<PF>(*reinterpret_cast<const VP *>(urow + v * VBP), w);
#pragma unroll
                                for (int i = 0; i < EPVP; i += 4) {
                                    const float4 tq = *reinterpret_cast<const float4 *>(te + v * EPVP + i);
                                    a = fmaf(w[i], tq.x, a);
                                    a = fmaf(w[i + 1], tq.y, a);
                                    a = fmaf(w[i + 2], tq.z, a);
                                    a = fmaf(w[i + 3], tq.w, a);
                                }
                            }
                        }
                        a = warp_sum(a);
                        if (lane == 0) {
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
        if (tid == 0) sm.nz_n = 0;
        cta_sync();
        cyc_b = clock64() - cb0;
        prof_put(p, li, 4, gtimer());

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

        // ---------------- phase C: gather rows of active neurons -------------
        const long long cc0 = clock64();
        const int m0 = sm.lst_n[0];
        const int m = m0 + (ntop > 1 ? sm.lst_n[1] : 0);
        // list index j -> (slot << 12 | local): slot 0 entries, then slot 1
        auto entry = [&](int j) -> int { return j < m0 ? sm.lst[j] : sm.lst[kMaxStrip + (j - m0)]; };
        const ExpertDev *exs[kMaxTopK] = {&p.ex[size_t(l) * p.E + sm.route_e[0]],
                                          &p.ex[size_t(l) * p.E + sm.route_e[ntop > 1 ? 1 : 0]]};
        for (int j = tid; j < m; j += kThreads) {
            const int en = entry(j), e = en >> 12, loc = en & 0xfff;
            prefetch_l2(exs[e]->Wgu + size_t(s0 + loc) * p.gu_bytes, uint32_t(p.gu_bytes));
            if (p.spec_down) prefetch_l2(exs[e]->Wd + size_t(s0 + loc) * p.wrow, uint32_t(p.wrow));
        }
        if (tid == kThreads - 1 && dense_ahead && l + 1 < l1) {
            const int ex[kMaxTopK] = {0, 0};
            prefetch_pred(l + 1, ex, true, true);
        }

        float acc[MAXVW * EPVW];
#pragma unroll
        for (int i = 0; i < MAXVW * EPVW; ++i) acc[i] = 0.f;

        const int nbat = (m + NB - 1) / NB;
        VW gv[NB][2][MAXVW];      // input records of the batch being loaded
        VW dv[NB][MAXVW];         // W_down rows being accumulated

        auto load_gu = [&](int bt) {
#pragma unroll
            for (int n = 0; n < NB; ++n) {
                const int j = bt * NB + n;
                if (j < m) {
                    const int en = entry(j), e = en >> 12, loc = en & 0xfff;
                    const uint8_t *rec = exs[e]->Wgu + size_t(s0 + loc) * p.gu_bytes;
#pragma unroll
                    for (int k = 0; k < MAXVW; ++k) {
                        const int v = tid + kThreads * k;
                        if (v < nvecW) {
                            gv[n][0][k] = ldvec<WF>(rec + v * VBW);
                            if (p.gated) gv[n][1][k] = ldvec<WF>(rec + p.wrow + v * VBW);
                        }
                    }
                }
            }
        };
        // dots of batch bt's records (in registers), reduced across the CTA;
        // neurons with h != 0 are appended to sm.nz in list order
        auto finish_gu = [&](int bt) {
            float pg[NB], pu[NB];
#pragma unroll
            for (int n = 0; n < NB; ++n) {
                pg[n] = 0.f;
                pu[n] = 0.f;
                const int j = bt * NB + n;
                if (j < m) {
                    const int en = entry(j), e = en >> 12, loc = en & 0xfff;
                    const uint8_t *rec = exs[e]->Wgu + size_t(s0 + loc) * p.gu_bytes;
#pragma unroll
                    for (int k = 0; k < MAXVW; ++k) {
                        const int v = tid + kThreads * k;
                        if (v < nvecW) {
                            float w[EPVW];
                            float a = 0.f;
                            cvt<WF>(gv[n][0][k], w);
#pragma unroll
                            for (int i = 0; i < EPVW; ++i) a = fmaf(w[i], xw[k * EPVW + i], a);
                            if constexpr (WF == kI4) a *= i4_scale(rec, d, v);
                            pg[n] += a;
                            if (p.gated) {
                                float c = 0.f;
                                cvt<WF>(gv[n][1][k], w);
#pragma unroll
                                for (int i = 0; i < EPVW; ++i) c = fmaf(w[i], xw[k * EPVW + i], c);
                                if constexpr (WF == kI4) c *= i4_scale(rec + p.wrow, d, v);
                                pu[n] += c;
                            }
                        }
                    }
                }
            }
#pragma unroll
            for (int n = 0; n < NB; ++n) {
                const float a = warp_sum(pg[n]);
                const float c = warp_sum(pu[n]);
                if (lane == 0) {
                    sm.red[rb][warp][2 * n] = a;
                    sm.red[rb][warp][2 * n + 1] = c;
                }
            }
            cta_sync();
            if (tid == 0) {
                int nzn = sm.nz_n;
                for (int n = 0; n < NB; ++n) {
                    const int j = bt * NB + n;
                    if (j >= m) break;
                    float G = 0.f, Uv = 0.f;
                    for (int w = 0; w < kConsumerWarps; ++w) {
                        G += sm.red[rb][w][2 * n];
                        Uv += sm.red[rb][w][2 * n + 1];
                    }
                    const int en = entry(j), e = en >> 12, loc = en & 0xfff;
                    const float h = act_h(p.act, G - sm.cbuf[e][loc], Uv) * sm.route_w[e];
                    if (h != 0.f) {
                        sm.nz[nzn] = int16_t(en);
                        sm.hz[nzn] = h;
                        ++nzn;
                    }
                }
                sm.nz_n = nzn;
            }
            cta_sync();
            rb ^= 1;
        };
        // W_down rows of sm.nz[q0, q1) into registers / into acc
        auto load_dn = [&](int q0, int q1) {
#pragma unroll
            for (int n = 0; n < NB; ++n) {
                const int q = q0 + n;
                if (q < q1) {
                    const int en = sm.nz[q], e = en >> 12, loc = en & 0xfff;
                    const uint8_t *row = exs[e]->Wd + size_t(s0 + loc) * p.wrow;
#pragma unroll
                    for (int k = 0; k < MAXVW; ++k) {
                        const int v = tid + kThreads * k;
                        if (v < nvecW) dv[n][k] = ldvec<WF>(row + v * VBW);
                    }
                }
            }
        };
        auto axpy_dn = [&](int q0, int q1) {
#pragma unroll
            for (int n = 0; n < NB; ++n) {
                const int q = q0 + n;
                if (q < q1) {
                    const int en = sm.nz[q], e = en >> 12, loc = en & 0xfff;
                    const uint8_t *row = exs[e]->Wd + size_t(s0 + loc) * p.wrow;
                    const float h = sm.hz[q];
#pragma unroll
                    for (int k = 0; k < MAXVW; ++k) {
                        const int v = tid + kThreads * k;
                        if (v < nvecW) {
                            float w[EPVW];
                            cvt<WF>(dv[n][k], w);
                            float hs = h;
                            if constexpr (WF == kI4) hs = h * i4_scale(row, d, v);
#pragma unroll
                            for (int i = 0; i < EPVW; ++i) acc[k * EPVW + i] = fmaf(hs, w[i], acc[k * EPVW + i]);
                        }
                    }
                }
            }
        };

        int dn_done = 0;   // entries of sm.nz already accumulated
        if (nbat > 0) {
            load_gu(0);
            finish_gu(0);
        }
        for (int bt = 0; bt < nbat; ++bt) {
            // W_down rows found so far + the records of batch bt + 1, together
            const int dn_hi = min(sm.nz_n, dn_done + NB);
            load_dn(dn_done, dn_hi);
            if (bt + 1 < nbat) load_gu(bt + 1);
            axpy_dn(dn_done, dn_hi);
            dn_done = dn_hi;
            if (bt + 1 < nbat) finish_gu(bt + 1);
        }
        const int nz_total = sm.nz_n;
        while (dn_done < nz_total) {
            const int dn_hi = min(nz_total, dn_done + NB);
            load_dn(dn_done, dn_hi);
            axpy_dn(dn_done, dn_hi);
            dn_done = dn_hi;
        }
        if (tid == 0 && p.stats) atomicAdd(p.stats + li * 4 + 1, nz_total);
        // per-CTA partial of y
#pragma unroll
        for (int k = 0; k < MAXVW; ++k) {
            const int v = tid + kThreads * k;
            if (v < nvecW) {
#pragma unroll
                for (int i = 0; i < EPVW; i += 4)
                    __stcg(reinterpret_cast<float4 *>(p.partials + size_t(b) * d + v * EPVW + i),
                           make_float4(acc[k * EPVW + i], acc[k * EPVW + i + 1],
                                       acc[k * EPVW + i + 2], acc[k * EPVW + i + 3]));
            }
        }
        cyc_c = clock64() - cc0;
        prof_put(p, li, 5, gtimer());
        prof_put(p, li, 6, gtimer());
        if (!grid_sync(&sm, p, epoch, bci, &cyc_bar)) break;
        prof_put(p, li, 7, gtimer());

        // ---------------- phase D: r += sum of partials (fixed order) --------
        {
            constexpr int kParts = kMaxStrips / 32;   // partial rows per lane
            const int nq = d / 4;
            const int q0 = int((long long)b * nq / S), q1 = int((long long)(b + 1) * nq / S);
            for (int q = q0 + warp; q < q1; q += kConsumerWarps) {
                float4 pv[kParts];
#pragma unroll
                for (int j = 0; j < kParts; ++j) {
                    const int c = lane + 32 * j;
                    pv[j] = c < S ? __ldcg(reinterpret_cast<const float4 *>(p.partials + size_t(c) * d) + q)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
                }
                float4 sacc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int j = 0; j < kParts; ++j) {
                    sacc.x += pv[j].x; sacc.y += pv[j].y; sacc.z += pv[j].z; sacc.w += pv[j].w;
                }
                sacc.x = warp_sum(sacc.x); sacc.y = warp_sum(sacc.y);
                sacc.z = warp_sum(sacc.z); sacc.w = warp_sum(sacc.w);
                if (lane == 0) {
                    float4 rv = __ldcg(reinterpret_cast<const float4 *>(p.resid) + q);
                    rv.x += sacc.x; rv.y += sacc.y; rv.z += sacc.z; rv.w += sacc.w;
                    __stcg(reinterpret_cast<float4 *>(p.resid) + q, rv);
                }
            }
        }
        prof_put(p, li, 8, gtimer());
        if (!grid_sync(&sm, p, epoch, bci, &cyc_bar)) break;
        prof_put(p, li, 9, gtimer());
        prof_put(p, li, 10, cyc_a);
        prof_put(p, li, 11, cyc_b);
        prof_put(p, li, 12, cyc_c);
        prof_put(p, li, 13, cyc_bar);
    }
}

template <int WF, int PF>
cudaError_t launch_t(int dmax_cls, const DecodeParams &p, cudaStream_t st, bool query, int *blocks)
{
    void *fn = nullptr;
    switch (dmax_cls) {
    case 0: fn = (void *)decode_kernel<WF, PF, 2048>; break;
    case 1: fn = (void *)decode_kernel<WF, PF, 4096>; break;
    default:
        if constexpr (WF == kF32 || PF == kF32) return cudaErrorInvalidValue;
        else fn = (void *)decode_kernel<WF, PF, 8192>;
        break;
    }
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kStageBytes);
    if (e != cudaSuccess) return e;
    if (query) return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks, fn, kThreads, kStageBytes);
    void *args[] = {const_cast<DecodeParams *>(&p)};
    return cudaLaunchCooperativeKernel(fn, dim3(p.S), dim3(kThreads), args, kStageBytes, st);
}

cudaError_t dispatch(int wfmt, int pfmt, int d, const DecodeParams *p, cudaStream_t st, bool query,
                     int *blocks)
{
    const int cls = d <= 2048 ? 0 : (d <= 4096 ? 1 : 2);
    static const DecodeParams dummy{};
    const DecodeParams &pp = p ? *p : dummy;
    if (wfmt == kF32 && pfmt == kF32) return launch_t<kF32, kF32>(cls, pp, st, query, blocks);
    if (wfmt == kF16 && pfmt == kF16) return launch_t<kF16, kF16>(cls, pp, st, query, blocks);
    if (wfmt == kBF16 && pfmt == kBF16) return launch_t<kBF16, kBF16>(cls, pp, st, query, blocks);
    if (wfmt == kI4 && pfmt == kF16) return launch_t<kI4, kF16>(cls, pp, st, query, blocks);
    if (wfmt == kI4 && pfmt == kBF16) return launch_t<kI4, kBF16>(cls, pp, st, query, blocks);
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode(int wfmt, int pfmt, const DecodeParams &p, cudaStream_t stream)
{
    return dispatch(wfmt, pfmt, p.d, &p, stream, false, nullptr);
}

int decode_max_blocks_per_sm(int wfmt, int pfmt, int d)
{
    int blocks = 0;
    if (dispatch(wfmt, pfmt, d, nullptr, nullptr, true, &blocks) != cudaSuccess) return 0;
    return blocks;
}

}  // namespace pi
