// pi_decode.cu -- persistent sparse-FFN decode kernel for sm_100a.
//
// One cooperative launch runs a range of layers for one token.  Each CTA owns
// one strip of the neuron table (a contiguous run of table positions holding
// a balanced share of hot neurons, hottest first).  Per layer:
//
//   phase A  x = RMSNorm(r) (every CTA, identical arithmetic); [MoE] router +
//            top-2 (every CTA, identical); rows [a0, a1) of t = V x.
//   --- grid barrier ---
//   phase B  z = U t - c for the CTA's strip; active iff z > threshold; the
//            active list is compacted in ascending table order with warp
//            ballots (PowerInfer (unite.ai), "Adaptive sparse predictor").
//   phase C  for active neurons only: rows of W_gate / W_up -> h = act(g, u);
//            for h != 0: the neuron's W_down column (stored as a row) is
//            accumulated into a per-CTA fp32 partial of y ("Neuron-aware
//            operators": rows of the input matrices, columns of the output).
//   --- grid barrier ---
//   phase D  r <- r + sum of the per-CTA partials, in fixed CTA order, by
//            column slices (deterministic; no atomics).  This is the merge of
//            the per-processor partial results (nearauto.com PowerInfer
//            article, Fig. 8), done in HBM-resident fp32 on one GPU.
//   --- grid barrier ---
//
// Warp roles: warps 0-7 compute.  Warp 8 streams the predictor weights (V rows
// of the CTA's t slice, U rows of its strip), which do not depend on the
// input, into a ring of 16 KB shared-memory slots with cp.async.bulk, running
// ahead across layers as far as the ring allows.  Warp 9 streams the rows of
// active neurons into a second ring: the gate/up rows as soon as the active
// list is known, each down row as soon as its h is known to be non-zero.
// Every slot carries a descriptor so consumers process the ring in issue
// order.  All waits are bounded (%globaltimer); a wait that runs out records
// an error word and every thread of the grid returns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "pi_internal.h"

namespace pi {
namespace {

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
__device__ __forceinline__ void mbar_arrive(uint64_t *b)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(s2u(b)) : "memory");
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
__device__ __forceinline__ uint64_t policy_evict_first()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
// 1-D bulk copy global -> this CTA's shared memory, completion on `bar`.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes,
                                         uint64_t *bar, uint64_t pol)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(s2u(dst)),
        "l"(src), "r"(bytes), "r"(s2u(bar)), "l"(pol)
        : "memory");
}
// Bulk prefetch of a global range into L2 (fire and forget), in 32 KB pieces.
__device__ __forceinline__ void prefetch_l2(const void *src, uint32_t bytes)
{
    const uint8_t *p = static_cast<const uint8_t *>(src);
    for (uint32_t o = 0; o < bytes; o += 32768u) {
        const uint32_t n = bytes - o < 32768u ? bytes - o : 32768u;
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p + o), "r"(n) : "memory");
    }
}
__device__ __forceinline__ long long gtimer()
{
    long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void cons_sync()
{
    asm volatile("bar.sync 1, 256;" ::: "memory");
}
__device__ __forceinline__ int ld_vol(const int *p)
{
    return *reinterpret_cast<const volatile int *>(p);
}
__device__ __forceinline__ void st_vol(int *p, int v)
{
    *reinterpret_cast<volatile int *>(p) = v;
}
__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned *p)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ unsigned atom_add_acqrel_gpu(unsigned *p, unsigned v)
{
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}
__device__ __forceinline__ void st_release_gpu(unsigned *p, unsigned v)
{
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// ---------------------------------------------------------------------------
// Stored formats: one vector = 16 bytes (8 bytes for INT4) of a row.
// ---------------------------------------------------------------------------
template <int F> struct Fm;
template <> struct Fm<kF32>  { static constexpr int VB = 16, EPV = 4; };
template <> struct Fm<kF16>  { static constexpr int VB = 16, EPV = 8; };
template <> struct Fm<kBF16> { static constexpr int VB = 16, EPV = 8; };
template <> struct Fm<kI4>   { static constexpr int VB = 8, EPV = 16; };

template <int F>
__device__ __forceinline__ void load_vec(const uint8_t *p, float *o)
{
    if constexpr (F == kF32) {
        float4 v = *reinterpret_cast<const float4 *>(p);
        o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
    } else if constexpr (F == kF16) {
        uint4 v = *reinterpret_cast<const uint4 *>(p);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __half2 h2 = *reinterpret_cast<const __half2 *>(&w[i]);
            float2 f = __half22float2(h2);
            o[2 * i] = f.x;
            o[2 * i + 1] = f.y;
        }
    } else if constexpr (F == kBF16) {
        uint4 v = *reinterpret_cast<const uint4 *>(p);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            o[2 * i] = __uint_as_float(w[i] << 16);
            o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    } else {
        // 16 nibbles, element 2j in the low nibble of byte j.  n - 8 is formed
        // exactly by placing n in the mantissa of 2^23 and subtracting 2^23 + 8.
        uint2 v = *reinterpret_cast<const uint2 *>(p);
        const uint32_t w[2] = {v.x, v.y};
#pragma unroll
        for (int i = 0; i < 2; ++i) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                uint32_t n = (w[i] >> (4 * j)) & 0xfu;
                o[8 * i + j] = __uint_as_float(0x4b000000u | n) - 8388616.0f;
            }
        }
    }
}

// Scale of the group holding vector v of an INT4 row record (nibbles, then
// one fp16 scale per 32 elements).
__device__ __forceinline__ float i4_scale(const uint8_t *row, int d, int v)
{
    return __half2float(*reinterpret_cast<const __half *>(row + d / 2 + (v >> 1) * 2));
}

// Partial dot product of a row (in shared memory) with this thread's cached
// x values.  Thread t owns vectors t, t + 256, ... of the row.
template <int F, int MAXV>
__device__ __forceinline__ float dot_row(const uint8_t *row, const float *xc, int nvec, int d)
{
    constexpr int EPV = Fm<F>::EPV, VB = Fm<F>::VB;
    float acc = 0.f;
#pragma unroll
    for (int k = 0; k < MAXV; ++k) {
        const int v = threadIdx.x + kConsumers * k;
        if (v < nvec) {
            float w[EPV];
            load_vec<F>(row + v * VB, w);
            float a = 0.f;
#pragma unroll
            for (int i = 0; i < EPV; ++i)
                a = fmaf(w[i], xc[k * EPV + i], a);
            if constexpr (F == kI4)
                acc = fmaf(i4_scale(row, d, v), a, acc);
            else
                acc += a;
        }
    }
    return acc;
}

// acc[owned columns] += h * row[owned columns]
template <int F, int MAXV>
__device__ __forceinline__ void axpy_row(const uint8_t *row, float h, float *acc, int nvec, int d)
{
    constexpr int EPV = Fm<F>::EPV, VB = Fm<F>::VB;
#pragma unroll
    for (int k = 0; k < MAXV; ++k) {
        const int v = threadIdx.x + kConsumers * k;
        if (v < nvec) {
            float w[EPV];
            load_vec<F>(row + v * VB, w);
            float hs = h;
            if constexpr (F == kI4)
                hs = h * i4_scale(row, d, v);
#pragma unroll
            for (int i = 0; i < EPV; ++i)
                acc[k * EPV + i] = fmaf(hs, w[i], acc[k * EPV + i]);
        }
    }
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float act_h(int act, float g, float u)
{
    const float gp = g > 0.f ? g : 0.f;
    if (act == 0) return gp;              // ReLU (non-gated)
    if (act == 1) return gp * u;          // ReGLU
    return gp * (u > 0.f ? u : 0.f);      // dReLU
}

// ---------------------------------------------------------------------------
// Shared-memory control block
// ---------------------------------------------------------------------------
enum GType { kGU = 0, kDown = 2 };   // a neuron's input record, or its W_down row
struct GDesc {
    int type, e, k;
    float h;
};
constexpr int kQueue = kMaxTopK * kMaxStrip;  // down-row request queue

struct Ctl {
    uint64_t p_full[kMaxPSlots], p_empty[kMaxPSlots];
    uint64_t g_full[kMaxGSlots], g_empty[kMaxGSlots];
    uint64_t route_ready, list_ready;
    GDesc gdesc[kMaxGSlots];
    int abort_flag;
    int bc[2];                                   // broadcast of collective decisions
    int route_e[2][kMaxTopK];                    // [layer parity][slot] expert id
    float route_w[2][kMaxTopK];
    int lst_n[2][kMaxTopK];
    int16_t lst[2][kMaxTopK][kMaxStrip];         // active strip-local indices, ascending
    int dq[kQueue];                              // down-row requests: (slot << 16) | k
    float dqh[kQueue];
    int dq_tail, h_rep;                          // cumulative counters (consumer thread 0)
    float zbuf[kMaxTopK][kMaxStrip];
    float cbuf[kMaxTopK][kMaxStrip];
    float tsm[kMaxRankTotal];
    float red[2][kConsumerWarps][17];
    float inv_rms;
    float logits[kMaxExperts];
};

}  // namespace

size_t decode_smem_bytes(int np_slots, int ng_slots, int sg_bytes)
{
    size_t ctl = (sizeof(Ctl) + 127) & ~size_t(127);
    return ctl + size_t(np_slots) * kPSlotBytes + size_t(ng_slots) * sg_bytes + 128;
}

namespace {

struct Piece {
    int kind;   // 0: V rows, 1: U rows
    int slot;   // expert slot (0 .. top_k-1)
    int row0;   // first row (V: within the expert's V; U: table position)
    int nrows;
};

__device__ __forceinline__ int make_pieces(int r, int ntop, int a0, int a1, int s0, int ns,
                                           Piece *pc)
{
    int n = 0;
    for (int e = 0; e < ntop; ++e) {
        const int lo = max(a0, e * r), hi = min(a1, (e + 1) * r);
        if (hi > lo) pc[n++] = Piece{0, e, lo - e * r, hi - lo};
    }
    for (int e = 0; e < ntop; ++e)
        if (ns > 0) pc[n++] = Piece{1, e, s0, ns};
    return n;
}

__device__ __forceinline__ void prof_mark(const DecodeParams &p, int li, int point)
{
    if (p.prof && threadIdx.x == 0)
        p.prof[(size_t(li) * kProfPoints + point) * gridDim.x + blockIdx.x] = gtimer();
}
__device__ __forceinline__ void prof_put(const DecodeParams &p, int li, int point, long long v)
{
    if (p.prof && threadIdx.x == 0)
        p.prof[(size_t(li) * kProfPoints + point) * gridDim.x + blockIdx.x] = v;
}

__device__ void set_error(int *err, int code)
{
    atomicCAS(err, 0, code);
}

// Bounded wait on an mbarrier phase by a single thread.  Returns false when
// the CTA is aborting or the wait ran out (which starts the abort).
__device__ bool wait_phase(uint64_t *bar, uint32_t parity, Ctl *ctl, const DecodeParams &p)
{
    if (mbar_test(bar, parity)) return true;
    const long long t0 = gtimer();
    for (unsigned it = 1;; ++it) {
        if (mbar_test(bar, parity)) return true;
        if ((it & 15) == 0) {
            if (ld_vol(&ctl->abort_flag)) return false;
            if (gtimer() - t0 > p.wait_ns) {
                st_vol(&ctl->abort_flag, 1);
                set_error(p.err, kDevTimeout);
                return false;
            }
        }
    }
}

// Collective wait of the 256 consumer threads: thread 0 waits (bounded) and
// broadcasts the outcome, so every consumer thread takes the same branch.
__device__ __forceinline__ bool cwait(uint64_t *bar, uint32_t parity, Ctl *ctl,
                                      const DecodeParams &p, int &bci, long long *wait_cyc = nullptr)
{
    if (threadIdx.x == 0) {
        const long long c0 = clock64();
        st_vol(&ctl->bc[bci], wait_phase(bar, parity, ctl, p) ? 1 : 0);
        if (wait_cyc) *wait_cyc += clock64() - c0;
    }
    cons_sync();
    const bool ok = ld_vol(&ctl->bc[bci]) != 0;
    bci ^= 1;
    if (ok) mbar_test(bar, parity);   // acquire for this thread (phase already complete)
    return ok;
}

// Grid-wide barrier of the consumer warps of all CTAs (one cooperative launch).
// bar[0] counts arrivals (never reset within a launch); the CTA whose arrival
// completes barrier `epoch` publishes it in bar[1]; the others wait for that
// generation word, so the waiting CTAs poll a line that changes once.
__device__ bool grid_sync(Ctl *ctl, const DecodeParams &p, unsigned &epoch, int &bci,
                          long long *wait_cyc = nullptr)
{
    cons_sync();
    const long long c0 = clock64();
    if (threadIdx.x == 0) {
        bool ok = ld_vol(&ctl->abort_flag) == 0;
        epoch += 1;
        if (ok) {
            unsigned last = epoch * gridDim.x - 1;
            if ((p.debug_flags & 1) && epoch == 1) last += 1;   // PI_DEBUG_STALL_BARRIER
            __threadfence();
            const unsigned old = atom_add_acqrel_gpu(p.bar, 1u);
            if (old == last) {
                st_release_gpu(p.bar + 1, epoch);
            } else {
                const long long t0 = gtimer();
                unsigned it = 0;
                while (ld_acquire_gpu(p.bar + 1) < epoch) {
                    if ((++it & 31) == 0) {
                        if (ld_vol(&ctl->abort_flag)) { ok = false; break; }
                        if (gtimer() - t0 > p.wait_ns) {
                            st_vol(&ctl->abort_flag, 1);
                            set_error(p.err, kDevTimeout);
                            ok = false;
                            break;
                        }
                    }
                }
            }
            __threadfence();
        }
        st_vol(&ctl->bc[bci], ok ? 1 : 0);
        if (wait_cyc) *wait_cyc += clock64() - c0;
    }
    cons_sync();
    const bool ok = ld_vol(&ctl->bc[bci]) != 0;
    bci ^= 1;
    return ok;
}

// Wait for every bulk copy this producer issued into a ring (used when the
// CTA aborts, so no copy is in flight when the CTA exits).
__device__ void drain_ring(uint64_t *full, int nslots, int issued, long long wait_ns)
{
    for (int s = 0; s < nslots && s < issued; ++s) {
        const int uses = (issued - 1 - s) / nslots + 1;
        const uint32_t par = (uses - 1) & 1;
        const long long t0 = gtimer();
        while (!mbar_test(&full[s], par))
            if (gtimer() - t0 > wait_ns) break;
    }
}

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------
template <int WF, int PF, int DMAX>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ DecodeParams p)
{
    constexpr int EPVW = Fm<WF>::EPV, EPVP = Fm<PF>::EPV;
    constexpr int MAXVW = (DMAX / EPVW + kConsumers - 1) / kConsumers;
    constexpr int MAXVP = (DMAX / EPVP + kConsumers - 1) / kConsumers;
    constexpr int MAXU = 4;                    // U vectors per lane (rank <= 128 * EPVP)
    // V rows per P slot at most: rows are >= 512 B below d = 2048, >= 4.5 KB up
    // to 4096 and >= 8.5 KB above
    constexpr int MAXRV = DMAX == 2048 ? 16 : (DMAX == 4096 ? 4 : 2);

    extern __shared__ __align__(128) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                                ~uintptr_t(127));
    Ctl *ctl = reinterpret_cast<Ctl *>(smem);
    uint8_t *pring = smem + ((sizeof(Ctl) + 127) & ~size_t(127));
    uint8_t *gring = pring + size_t(p.np_slots) * kPSlotBytes;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.x, S = gridDim.x;
    const int d = p.d, r = p.r, NP = p.np_slots, NG = p.ng_slots, SG = p.sg_bytes;
    const int s0 = p.strip_off[b], ns = p.strip_off[b + 1] - s0;
    const bool predict = p.mode == kModePredict;
    const int ntop = predict ? 1 : p.top_k;
    const int rows_total = ntop * r;
    const int a0 = int((long long)b * rows_total / S), a1 = int((long long)(b + 1) * rows_total / S);
    const int RV = min(MAXRV, kPSlotBytes / p.vrow), RU = kPSlotBytes / p.urow;
    const int nvecW = (WF == kI4 ? d / 2 : d * (WF == kF32 ? 4 : 2)) / Fm<WF>::VB;
    const int nvecP = p.vrow / Fm<PF>::VB;
    const int nvecU = p.urow / Fm<PF>::VB;
    const int l0 = predict ? p.layer_begin : p.layer_begin;
    const int l1 = predict ? p.layer_begin + 1 : p.layer_end;

    if (tid == 0) {
        for (int i = 0; i < NP; ++i) {
            mbar_init(&ctl->p_full[i], 1);
            mbar_init(&ctl->p_empty[i], kConsumerWarps);
        }
        for (int i = 0; i < NG; ++i) {
            mbar_init(&ctl->g_full[i], 1);
            mbar_init(&ctl->g_empty[i], kConsumerWarps);
        }
        mbar_init(&ctl->route_ready, 1);
        mbar_init(&ctl->list_ready, 1);
        ctl->abort_flag = 0;
        ctl->dq_tail = 0;
        ctl->h_rep = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    // =====================================================================
    // Warp 8: predictor stream (V rows of the t slice, U rows of the strip)
    // =====================================================================
    if (warp == kPWarp) {
        if (lane != 0) return;
        const uint64_t pol = policy_evict_first();
        int pi = 0;
        bool ok = true;
        // L2 prefetch of all predictor bytes a layer will stream into this CTA
        auto prefetch_layer = [&](int l, const int *experts) {
            Piece pc[2 * kMaxTopK];
            const int npc = make_pieces(r, ntop, a0, a1, s0, ns, pc);
            for (int q = 0; q < npc; ++q) {
                const ExpertDev &ex = p.ex[size_t(l) * p.E + experts[pc[q].slot]];
                const int rowb = pc[q].kind == 0 ? p.vrow : p.urow;
                const uint8_t *base = pc[q].kind == 0 ? ex.V : ex.U;
                prefetch_l2(base + size_t(pc[q].row0) * rowb, uint32_t(pc[q].nrows) * rowb);
            }
        };
        const bool dense_ahead = !predict && p.E == 1;   // experts known ahead of time
        if (dense_ahead) {
            const int e0[kMaxTopK] = {0, 0};
            prefetch_layer(l0, e0);
        }
        for (int l = l0; l < l1 && ok; ++l) {
            const int lp = (l - l0) & 1;
            int experts[kMaxTopK] = {0, 0};
            if (predict) {
                experts[0] = p.pred_expert;
                prefetch_layer(l, experts);
            } else if (p.E > 1) {
                if (!wait_phase(&ctl->route_ready, (l - l0) & 1, ctl, p)) { ok = false; break; }
                experts[0] = ctl->route_e[lp][0];
                experts[1] = ctl->route_e[lp][1];
                prefetch_layer(l, experts);
            }
            Piece pc[2 * kMaxTopK];
            const int npc = make_pieces(r, ntop, a0, a1, s0, ns, pc);
            for (int q = 0; q < npc && ok; ++q) {
                const ExpertDev &ex = p.ex[size_t(l) * p.E + experts[pc[q].slot]];
                const int rowb = pc[q].kind == 0 ? p.vrow : p.urow;
                const int per = pc[q].kind == 0 ? RV : RU;
                const uint8_t *base = pc[q].kind == 0 ? ex.V : ex.U;
                for (int row = 0; row < pc[q].nrows; row += per) {
                    const int n = min(per, pc[q].nrows - row);
                    const int s = pi % NP;
                    if (!wait_phase(&ctl->p_empty[s], ((pi / NP) & 1) ^ 1, ctl, p)) { ok = false; break; }
                    const uint32_t bytes = uint32_t(n) * rowb;
                    mbar_arrive_tx(&ctl->p_full[s], bytes);
                    bulk_g2s(pring + size_t(s) * kPSlotBytes,
                             base + size_t(pc[q].row0 + row) * rowb, bytes, &ctl->p_full[s], pol);
                    ++pi;
                }
            }
            if (ok && dense_ahead && l + 1 < l1) {
                const int e0[kMaxTopK] = {0, 0};
                prefetch_layer(l + 1, e0);
            }
        }
        if (!ok) drain_ring(ctl->p_full, NP, pi, p.wait_ns);
        return;
    }

    // =====================================================================
    // Warp 9: gather stream (rows of active neurons)
    // =====================================================================
    if (warp == kGWarp) {
        if (lane != 0 || predict) return;
        const uint64_t pol = policy_evict_first();
        int gi = 0, rep_base = 0, dq_head = 0;
        bool ok = true;
        auto issue = [&](int type, int e, int k, float h, const uint8_t *src, int bytes) -> bool {
            const int s = gi % NG;
            if (!wait_phase(&ctl->g_empty[s], ((gi / NG) & 1) ^ 1, ctl, p)) return false;
            ctl->gdesc[s] = GDesc{type, e, k, h};
            mbar_arrive_tx(&ctl->g_full[s], uint32_t(bytes));
            bulk_g2s(gring + size_t(s) * SG, src, uint32_t(bytes), &ctl->g_full[s], pol);
            ++gi;
            return true;
        };
        for (int l = l0; l < l1 && ok; ++l) {
            const int lp = (l - l0) & 1;
            if (!wait_phase(&ctl->list_ready, (l - l0) & 1, ctl, p)) { ok = false; break; }
            const int m0 = ctl->lst_n[lp][0];
            const int m = m0 + (ntop > 1 ? ctl->lst_n[lp][1] : 0);
            const int ex0 = p.E > 1 ? ctl->route_e[lp][0] : 0;
            const int ex1 = p.E > 1 ? ctl->route_e[lp][1] : 0;
            const ExpertDev *exs[2] = {&p.ex[size_t(l) * p.E + ex0], &p.ex[size_t(l) * p.E + ex1]};
            // every row this CTA may need this layer starts moving towards L2 now
            for (int j = 0; j < m; ++j) {
                const int e = j < m0 ? 0 : 1;
                const int k = ctl->lst[lp][e][j < m0 ? j : j - m0];
                prefetch_l2(exs[e]->Wgu + size_t(s0 + k) * p.gu_bytes, uint32_t(p.gu_bytes));
                if (p.spec_down)
                    prefetch_l2(exs[e]->Wd + size_t(s0 + k) * p.wrow, uint32_t(p.wrow));
            }
            const int rep_target = rep_base + m;
            int gu = 0;
            long long idle_since = gtimer();
            while (ok) {
                const int tail = ld_vol(&ctl->dq_tail);
                if (dq_head < tail) {
                    const int q = dq_head % kQueue;
                    const int ent = ld_vol(&ctl->dq[q]);
                    const float h = *reinterpret_cast<volatile float *>(&ctl->dqh[q]);
                    ++dq_head;
                    const int e = ent >> 16, k = ent & 0xffff;
                    ok = issue(kDown, e, k, h, exs[e]->Wd + size_t(s0 + k) * p.wrow, p.wrow);
                    idle_since = gtimer();
                } else if (gu < m) {
                    const int e = gu < m0 ? 0 : 1;
                    const int k = ctl->lst[lp][e][gu < m0 ? gu : gu - m0];
                    ++gu;
                    ok = issue(kGU, e, k, 0.f, exs[e]->Wgu + size_t(s0 + k) * p.gu_bytes, p.gu_bytes);
                    idle_since = gtimer();
                } else {
                    if (ld_vol(&ctl->h_rep) >= rep_target) {
                        __threadfence_block();
                        if (dq_head >= ld_vol(&ctl->dq_tail)) break;
                        continue;
                    }
                    if (ld_vol(&ctl->abort_flag)) { ok = false; break; }
                    if (gtimer() - idle_since > p.wait_ns) {
                        st_vol(&ctl->abort_flag, 1);
                        set_error(p.err, kDevTimeout);
                        ok = false;
                        break;
                    }
                }
            }
            rep_base = rep_target;
        }
        if (!ok) drain_ring(ctl->g_full, NG, gi, p.wait_ns);
        return;
    }

    // =====================================================================
    // Warps 0-7: arithmetic
    // =====================================================================
    unsigned epoch = 0;
    int bci = 0, pc_i = 0, gs = 0, rb = 0;
    int rep_count = 0, q_tail = 0;                 // thread 0's cumulative counters
    float xw[MAXVW * EPVW];
    float xp[MAXVP * EPVP];

    for (int l = l0; l < l1; ++l) {
        const int lp = (l - l0) & 1;
        const int li = l - l0;

        // ---------------- phase A: layer input, routing, t = V x ----------
        prof_mark(p, li, 0);
        long long wc_a = 0, wc_b = 0, wc_c = 0, wc_bar = 0;
        float inv = 1.f;
        const float *src = predict ? p.x_in : p.resid;
        // one round trip to L2: this thread's columns in both row formats
#pragma unroll
        for (int k = 0; k < MAXVW; ++k) {
            const int v = tid + kConsumers * k;
#pragma unroll
            for (int i = 0; i < EPVW; i += 4) {
                float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
                if (v < nvecW) q = __ldcg(reinterpret_cast<const float4 *>(src + v * EPVW + i));
                xw[k * EPVW + i] = q.x; xw[k * EPVW + i + 1] = q.y;
                xw[k * EPVW + i + 2] = q.z; xw[k * EPVW + i + 3] = q.w;
            }
        }
#pragma unroll
        for (int k = 0; k < MAXVP; ++k) {
            const int v = tid + kConsumers * k;
#pragma unroll
            for (int i = 0; i < EPVP; i += 4) {
                float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
                if (v < nvecP) q = __ldcg(reinterpret_cast<const float4 *>(src + v * EPVP + i));
                xp[k * EPVP + i] = q.x; xp[k * EPVP + i + 1] = q.y;
                xp[k * EPVP + i + 2] = q.z; xp[k * EPVP + i + 3] = q.w;
            }
        }
        if (!predict) {
            // x = r / sqrt(mean(r^2) + eps); the W-format columns cover d once
            float ss = 0.f;
#pragma unroll
            for (int k = 0; k < MAXVW; ++k) {
                const int v = tid + kConsumers * k;
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
            if (lane == 0) ctl->red[rb][warp][16] = ss;
            cons_sync();
            if (tid == 0) {
                float tot = 0.f;
                for (int w = 0; w < kConsumerWarps; ++w) tot += ctl->red[rb][w][16];
                ctl->inv_rms = 1.f / sqrtf(tot / float(d) + p.eps);
            }
            cons_sync();
            inv = ctl->inv_rms;
            rb ^= 1;
#pragma unroll
            for (int i = 0; i < MAXVW * EPVW; ++i) xw[i] *= inv;
#pragma unroll
            for (int i = 0; i < MAXVP * EPVP; ++i) xp[i] *= inv;
        }

        // MoE routing, computed identically by every CTA: logits of the E
        // experts (fp16 router), softmax, two largest (ties: lower index),
        // weights renormalised over the two, experts in ascending index.
        if (!predict && p.E > 1) {
            const __half *R = reinterpret_cast<const __half *>(p.router[l]);
            for (int e = 0; e < p.E; ++e) {
                float a = 0.f;
                for (int j = tid; j < d; j += kConsumers)
                    a = fmaf(__half2float(R[size_t(e) * d + j]), __ldcg(src + j) * inv, a);
                a = warp_sum(a);
                if (lane == 0) ctl->red[rb][warp][e] = a;
            }
            cons_sync();
            if (tid == 0) {
                float mx = -INFINITY;
                for (int e = 0; e < p.E; ++e) {
                    float s = 0.f;
                    for (int w = 0; w < kConsumerWarps; ++w) s += ctl->red[rb][w][e];
                    ctl->logits[e] = s;
                    mx = fmaxf(mx, s);
                }
                float pr[kMaxExperts];
                float den = 0.f;
                for (int e = 0; e < p.E; ++e) { pr[e] = expf(ctl->logits[e] - mx); den += pr[e]; }
                for (int e = 0; e < p.E; ++e) pr[e] /= den;
                int ea = 0;
                for (int e = 1; e < p.E; ++e) if (pr[e] > pr[ea]) ea = e;
                int eb = ea == 0 ? 1 : 0;
                for (int e = 0; e < p.E; ++e) if (e != ea && pr[e] > pr[eb]) eb = e;
                const int lo = min(ea, eb), hi = max(ea, eb);
                ctl->route_e[lp][0] = lo;
                ctl->route_e[lp][1] = hi;
                ctl->route_w[lp][0] = pr[lo] / (pr[lo] + pr[hi]);
                ctl->route_w[lp][1] = pr[hi] / (pr[lo] + pr[hi]);
                if (p.stats && b == 0) {
                    p.stats[li * 4 + 2] = lo;
                    p.stats[li * 4 + 3] = hi;
                }
                mbar_arrive(&ctl->route_ready);
            }
            cons_sync();
            rb ^= 1;
        } else if (tid == 0) {
            ctl->route_e[lp][0] = predict ? p.pred_expert : 0;
            ctl->route_e[lp][1] = 0;
            ctl->route_w[lp][0] = 1.f;
            ctl->route_w[lp][1] = 0.f;
            if (p.stats && b == 0 && !predict) {
                p.stats[li * 4 + 2] = -1;
                p.stats[li * 4 + 3] = -1;
            }
        }

        // t rows [a0, a1): consume the V chunks of the P ring
        prof_mark(p, li, 1);
        bool alive = true;
        {
            Piece pc[2 * kMaxTopK];
            const int npc = make_pieces(r, ntop, a0, a1, s0, ns, pc);
            for (int q = 0; q < npc && alive; ++q) {
                if (pc[q].kind != 0) continue;
                for (int row = 0; row < pc[q].nrows; row += RV) {
                    const int n = min(RV, pc[q].nrows - row);
                    const int s = pc_i % NP;
                    if (!cwait(&ctl->p_full[s], (pc_i / NP) & 1, ctl, p, bci, &wc_a)) { alive = false; break; }
                    const uint8_t *slot = pring + size_t(s) * kPSlotBytes;
                    float part[MAXRV];
#pragma unroll
                    for (int rr = 0; rr < MAXRV; ++rr)
                        part[rr] = rr < n ? dot_row<PF, MAXVP>(slot + rr * p.vrow, xp, nvecP, d) : 0.f;
#pragma unroll
                    for (int rr = 0; rr < MAXRV; ++rr) {
                        if (rr < n) {
                            const float v = warp_sum(part[rr]);
                            if (lane == 0) ctl->red[rb][warp][rr] = v;
                        }
                    }
                    cons_sync();
                    if (lane == 0) mbar_arrive(&ctl->p_empty[s]);
                    if (tid < n) {
                        float t = 0.f;
                        for (int w = 0; w < kConsumerWarps; ++w) t += ctl->red[rb][w][tid];
                        __stcg(p.t_buf + pc[q].slot * r + pc[q].row0 + row + tid, t);
                    }
                    rb ^= 1;
                    ++pc_i;
                }
            }
        }
        prof_mark(p, li, 2);
        if (!alive || !grid_sync(ctl, p, epoch, bci, &wc_bar)) break;
        prof_mark(p, li, 3);

        // ---------------- phase B: z = U t - c, threshold, compaction -----
        for (int i = tid; i < ntop * r; i += kConsumers) ctl->tsm[i] = __ldcg(p.t_buf + i);
        for (int e = 0; e < ntop; ++e) {
            const ExpertDev &ex = p.ex[size_t(l) * p.E + ctl->route_e[lp][e]];
            for (int i = tid; i < ns; i += kConsumers) ctl->cbuf[e][i] = __ldg(ex.c + s0 + i);
        }
        cons_sync();
        for (int e = 0; e < ntop && alive; ++e) {
            float tu[MAXU * EPVP];
#pragma unroll
            for (int k = 0; k < MAXU; ++k) {
                const int v = lane + 32 * k;
#pragma unroll
                for (int i = 0; i < EPVP; ++i)
                    tu[k * EPVP + i] = v < nvecU ? ctl->tsm[e * r + v * EPVP + i] : 0.f;
            }
            for (int row = 0; row < ns; row += RU) {
                const int n = min(RU, ns - row);
                const int s = pc_i % NP;
                if (!cwait(&ctl->p_full[s], (pc_i / NP) & 1, ctl, p, bci, &wc_b)) { alive = false; break; }
                const uint8_t *slot = pring + size_t(s) * kPSlotBytes;
                for (int rr = warp; rr < n; rr += kConsumerWarps) {
                    const uint8_t *urow = slot + size_t(rr) * p.urow;
                    float a = 0.f;
#pragma unroll
                    for (int k = 0; k < MAXU; ++k) {
                        const int v = lane + 32 * k;
                        if (v < nvecU) {
                            float w[EPVP];
                            load_vec<PF>(urow + v * Fm<PF>::VB, w);
#pragma unroll
                            for (int i = 0; i < EPVP; ++i) a = fmaf(w[i], tu[k * EPVP + i], a);
                        }
                    }
                    a = warp_sum(a);
                    if (lane == 0) {
                        const int loc = row + rr;
                        const float z = a - ctl->cbuf[e][loc];
                        ctl->zbuf[e][loc] = z;
                        if (predict && p.z_out) p.z_out[s0 + loc] = z;
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->p_empty[s]);
                ++pc_i;
            }
        }
        if (!alive) break;
        cons_sync();
        prof_mark(p, li, 4);
        // compaction in ascending strip order: warp e builds expert slot e's list
        if (warp < ntop) {
            const int e = warp;
            int cnt = 0;
            for (int base = 0; base < ns; base += 32) {
                const int loc = base + lane;
                const bool act = loc < ns && ctl->zbuf[e][loc] > p.threshold;
                const unsigned m = __ballot_sync(0xffffffffu, act);
                if (act) {
                    const int pos = cnt + __popc(m & ((1u << lane) - 1u));
                    ctl->lst[lp][e][pos] = int16_t(loc);
                    if (predict) p.lists[size_t(b) * kMaxStrip + pos] = s0 + loc;
                    if (p.masks) {
                        const int gp = s0 + loc;
                        const int words = (p.F + 31) / 32;
                        atomicOr(p.masks + (size_t(li) * ntop + e) * words + (gp >> 5), 1u << (gp & 31));
                    }
                }
                cnt += __popc(m);
            }
            if (lane == 0) {
                ctl->lst_n[lp][e] = cnt;
                if (predict) p.counts[b] = cnt;
                if (p.stats && !predict) atomicAdd(p.stats + li * 4 + 0, cnt);
            }
        }
        cons_sync();

        if (predict) {
            // global ascending list: prefix of the strip counts, then copy
            if (!grid_sync(ctl, p, epoch, bci)) break;
            int pre = 0;
            for (int i = tid; i < b; i += kConsumers) pre += __ldcg(p.counts + i);
            pre = __reduce_add_sync(0xffffffffu, pre);
            if (lane == 0) ctl->red[rb][warp][0] = __int_as_float(pre);
            cons_sync();
            int base = 0;
            for (int w = 0; w < kConsumerWarps; ++w) base += __float_as_int(ctl->red[rb][w][0]);
            const int cnt = ctl->lst_n[lp][0];
            for (int i = tid; i < cnt; i += kConsumers)
                p.idx_out[base + i] = s0 + ctl->lst[lp][0][i];
            if (b == S - 1 && tid == 0) p.count_out[0] = base + cnt;
            break;
        }

        if (tid == 0) mbar_arrive(&ctl->list_ready);
        prof_mark(p, li, 5);

        // ---------------- phase C: gather rows of active neurons ----------
        float acc[MAXVW * EPVW];
#pragma unroll
        for (int i = 0; i < MAXVW * EPVW; ++i) acc[i] = 0.f;
        {
            const int m = ctl->lst_n[lp][0] + (ntop > 1 ? ctl->lst_n[lp][1] : 0);
            const int cap = (p.gated ? 3 : 2) * m + 1;   // slots this layer can hold at most
            int gu_done = 0, dn_done = 0, nnz = 0;
            for (int iter = 0; (gu_done < m || dn_done < nnz) && iter < cap; ++iter) {
                const int s = gs % NG;
                if (!cwait(&ctl->g_full[s], (gs / NG) & 1, ctl, p, bci, &wc_c)) { alive = false; break; }
                const GDesc dsc = ctl->gdesc[s];
                const uint8_t *row = gring + size_t(s) * SG;
                if (dsc.type == kDown) {
                    axpy_row<WF, MAXVW>(row, dsc.h, acc, nvecW, d);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&ctl->g_empty[s]);
                    ++gs;
                    ++dn_done;
                    continue;
                }
                // the neuron's input record: gate (or W_1) row, then its up row
                float pg = dot_row<WF, MAXVW>(row, xw, nvecW, d);
                float pu = 0.f;
                if (p.gated) pu = dot_row<WF, MAXVW>(row + p.wrow, xw, nvecW, d);
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->g_empty[s]);
                ++gs;
                pg = warp_sum(pg);
                pu = warp_sum(pu);
                if (lane == 0) {
                    ctl->red[rb][warp][0] = pg;
                    ctl->red[rb][warp][1] = pu;
                }
                cons_sync();
                float G = 0.f, Uv = 0.f;
                for (int w = 0; w < kConsumerWarps; ++w) {
                    G += ctl->red[rb][w][0];
                    Uv += ctl->red[rb][w][1];
                }
                rb ^= 1;
                const int e = dsc.e & 1, k = dsc.k;
                const float g = G - ctl->cbuf[e][k];
                const float h = act_h(p.act, g, Uv) * ctl->route_w[lp][e];
                if (h != 0.f) ++nnz;
                if (tid == 0) {
                    if (h != 0.f) {
                        const int q = q_tail % kQueue;
                        ctl->dq[q] = (e << 16) | k;
                        ctl->dqh[q] = h;
                        __threadfence_block();
                        ++q_tail;
                        st_vol(&ctl->dq_tail, q_tail);
                    }
                    __threadfence_block();
                    ++rep_count;
                    st_vol(&ctl->h_rep, rep_count);
                }
                ++gu_done;
            }
            if (tid == 0 && p.stats) atomicAdd(p.stats + li * 4 + 1, nnz);
        }
        if (!alive) break;
        prof_mark(p, li, 6);
        // per-CTA partial of y
#pragma unroll
        for (int k = 0; k < MAXVW; ++k) {
            const int v = tid + kConsumers * k;
            if (v < nvecW) {
#pragma unroll
                for (int i = 0; i < EPVW; i += 4)
                    __stcg(reinterpret_cast<float4 *>(p.partials + size_t(b) * d + v * EPVW + i),
                           make_float4(acc[k * EPVW + i], acc[k * EPVW + i + 1],
                                       acc[k * EPVW + i + 2], acc[k * EPVW + i + 3]));
            }
        }
        if (!grid_sync(ctl, p, epoch, bci, &wc_bar)) break;
        prof_mark(p, li, 7);

        // ---------------- phase D: r += sum of partials (fixed order) -----
        {
            const int nq = d / 4;
            const int q0 = int((long long)b * nq / S), q1 = int((long long)(b + 1) * nq / S);
            for (int q = q0 + warp; q < q1; q += kConsumerWarps) {
                float4 sacc = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int c = lane; c < S; c += 32) {
                    const float4 v = __ldcg(reinterpret_cast<const float4 *>(p.partials + size_t(c) * d) + q);
                    sacc.x += v.x; sacc.y += v.y; sacc.z += v.z; sacc.w += v.w;
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
        prof_mark(p, li, 8);
        if (!grid_sync(ctl, p, epoch, bci, &wc_bar)) break;
        prof_mark(p, li, 9);
        prof_put(p, li, 10, wc_a);
        prof_put(p, li, 11, wc_b);
        prof_put(p, li, 12, wc_c);
        prof_put(p, li, 13, wc_bar);
    }
}

template <int WF, int PF>
cudaError_t launch_t(int dmax_cls, const DecodeParams &p, size_t smem, cudaStream_t st,
                     bool query, int *blocks)
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
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    if (query) return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks, fn, kThreads, smem);
    void *args[] = {const_cast<DecodeParams *>(&p)};
    return cudaLaunchCooperativeKernel(fn, dim3(p.S), dim3(kThreads), args, smem, st);
}

cudaError_t dispatch(int wfmt, int pfmt, int d, const DecodeParams *p, size_t smem,
                     cudaStream_t st, bool query, int *blocks)
{
    const int cls = d <= 2048 ? 0 : (d <= 4096 ? 1 : 2);
    static const DecodeParams dummy{};
    const DecodeParams &pp = p ? *p : dummy;
    if (wfmt == kF32 && pfmt == kF32) return launch_t<kF32, kF32>(cls, pp, smem, st, query, blocks);
    if (wfmt == kF16 && pfmt == kF16) return launch_t<kF16, kF16>(cls, pp, smem, st, query, blocks);
    if (wfmt == kBF16 && pfmt == kBF16) return launch_t<kBF16, kBF16>(cls, pp, smem, st, query, blocks);
    if (wfmt == kI4 && pfmt == kF16) return launch_t<kI4, kF16>(cls, pp, smem, st, query, blocks);
    if (wfmt == kI4 && pfmt == kBF16) return launch_t<kI4, kBF16>(cls, pp, smem, st, query, blocks);
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode(int wfmt, int pfmt, const DecodeParams &p, size_t smem, cudaStream_t stream)
{
    return dispatch(wfmt, pfmt, p.d, &p, smem, stream, false, nullptr);
}

int decode_max_blocks_per_sm(int wfmt, int pfmt, int d, size_t smem)
{
    int blocks = 0;
    if (dispatch(wfmt, pfmt, d, nullptr, smem, nullptr, true, &blocks) != cudaSuccess) return 0;
    return blocks;
}

}  // namespace pi
