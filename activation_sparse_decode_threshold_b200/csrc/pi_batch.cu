// pi_batch.cu -- small-batch sparse FFN decode (up to 8 independent tokens per
// launch) for sm_100a.
//
// The sparse path keeps its advantage at small batch sizes (nearauto.com
// PowerInfer article, "Experiments", Fig. 14).  With several tokens in one
// launch the rows that are read are those of the UNION of the tokens'
// predicted sets: each union neuron's W_gate / W_up / W_down rows are fetched
// once for the whole batch, and token b keeps its own predicted set (its h is
// exactly 0 outside it), so each token's output is its batch-1 output up to
// rounding.  The grid barriers and the predictor bytes are paid once per layer
// for all tokens.
//
// One cooperative launch per call, one CTA per strip, 16 warps.  Per layer:
//   [A] x_b = RMSNorm(r_b) for every token (the per-CTA sums of squares of
//       the column phase, summed in fixed order), kept in shared memory as
//       16-bit values for the tensor cores: F16 keeps x_hi (the gate/up
//       operand) and a remainder x_lo beside it for the predictor; BF16 keeps
//       both parts as operands everywhere (four tokens per launch, each
//       token's two parts in two columns of the mma tile); rows [a0, a1) of
//       t_b = V x_b by tensor-core dots over both parts.      --- barrier ---
//   [B] z_b = U t_b - c over the strip (tensor-core dots, t_b carried as
//       16-bit parts), per-neuron token masks, the union compacted in
//       ascending table order and published.                   --- barrier ---
//   [C] an equal share of the union per CTA; rounds of up to five neurons
//       whose gate|up|down rows arrive by bulk copy; G = W_gu X^T and
//       Y^T += W_d^T H by mma.sync (fp32 accumulators; F16: X and H rounded
//       to fp16, as in the dense prefill; BF16: X and H as two bf16 parts);
//       per-CTA partials of y for every token.                 --- barrier ---
//   [column phase] r_b += sum of the partials over CTAs in fixed order for
//       this CTA's columns; per-CTA sums of squares.          --- barrier ---
// Dense FFN layers with F16 or BF16 weights and predictor, d_model <= 4096.
// Every wait is bounded (%globaltimer); a wait that runs out records an error
// word and the CTA leaves after draining its copies.
#include "pi_decode_kernel.cuh"

namespace pi {

namespace {

constexpr int kNB = 8;                  // columns of one mma tile: tokens x parts per launch
constexpr int kBD = 4096;               // d_model at most
constexpr int kBRound = 5;              // union neurons per gather round at most
constexpr int kXBytes = kNB * kBD * 2;  // x of every token, 16-bit
constexpr int kBStage = 128 * 1024;     // staging: V rows + x remainders / t parts + U rows / records
constexpr int kTPartBytes = 52 * 1024;  // t parts (phase B), at the start of the staging buffer
constexpr int kGredFloats = kConsumerWarps * 16 * kNB * 2;   // cross-warp gate/up sums of a round
constexpr int kBSmem = kXBytes + kBStage + kGredFloats * 4;  // dynamic shared memory

struct BatchParams {
    const ExpertDev *ex;        // [n_layers] (dense)
    const uint8_t *const *vrm;  // [n_layers] V row-major (r x vrow bytes)
    const int32_t *strip_off;   // [S + 1]
    const int32_t *grp_off;     // [S + 1] column slices in 8-column groups
    int d, F, r, act, gated, S, nb;
    int layer_begin, layer_end;
    float threshold, eps;
    int vrow, urow, wrow, gu_bytes, rec_bytes, wd_stride, spec, u_swz;
    float *resid;               // [nb x d] in/out
    float *trace;               // [(l1 - l0) x ntok x d] or null: rows tok0 .. tok0 + nb - 1
    int32_t *stats;             // [(l1 - l0) x 4] or null (zeroed by the host)
    uint32_t *masks;            // [(l1 - l0) x ntok x ceil(F/32)] or null (zeroed)
    int ntok, tok0;             // tokens of the whole call, first token of this launch
    float *t_buf;               // [nb x r]
    float *ss;                  // [S x kNB] per-CTA sums of squares
    float *partials;            // [S x nb x d]
    int32_t *counts;            // [S]
    unsigned long long *pub;    // [S x kMaxStrip] union entries: (mask << 24 | pos) | bias << 32
    unsigned *bar;              // grid barrier counters (zeroed before launch)
    int *err;
    long long wait_ns;
};

struct BSmem {
    int32_t glst[kMaxTopK * kMaxStrip];    // this CTA's share of the union: (mask << 24) | position
    float gc[kMaxTopK * kMaxStrip];        // their biases
    uint32_t zmask[kMaxStrip];             // token mask of each strip neuron (phase B)
    float cbuf[kMaxStrip];                 // strip biases
    int32_t lst[kMaxStrip];                // union of the strip: table positions
    int scan[kMaxStrips + 1];
    int red[kConsumerWarps];
    float inv[kNB];
    alignas(16) uint16_t hs[kNB][16];      // H of a round: [token][slot], weight format
    alignas(16) float rsl[kNB][kMaxSliceCols / 4];   // column phase: this CTA's columns of each token's r
    int lst_n, share_n, nzu;
    int bc[2];
    uint64_t bar_v, bar_u, bar_g;
};
static_assert(kMaxSliceCols / 4 >= 256, "column slice of one token in the column phase");

template <int F>
__device__ __forceinline__ uint16_t to16(float v)
{
    if constexpr (F == kBF16) return __bfloat16_as_ushort(__float2bfloat16_rn(v));
    else return __half_as_ushort(__float2half_rn(v));
}
template <int F>
__device__ __forceinline__ float from16(uint16_t v)
{
    if constexpr (F == kBF16) return __uint_as_float(uint32_t(v) << 16);
    else return __half2float(__ushort_as_half(v));
}

// byte offset of element j of token row t in the x arrays: rows of d 16-bit
// values, 16-byte chunks permuted inside each 128-byte group by the token
// index (so the 8 token rows of a matrix load hit 8 different bank groups)
__device__ __forceinline__ uint32_t xoff(int t, int j, int d)
{
    const int c = j >> 3;
    return uint32_t(t * d * 2 + (((c & ~7) | ((c ^ t) & 7)) << 4) + (j & 7) * 2);
}

// Four 8x8 b16 matrices, transposed on the way.
__device__ __forceinline__ void ldsm_x4_t(const void *p, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(s2u(p)));
}
__device__ __forceinline__ void ldsm_x2(const void *p, uint32_t &r0, uint32_t &r1)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
                 : "=r"(r0), "=r"(r1)
                 : "r"(s2u(p)));
}

// grid barrier in two halves (arrival, then a bounded wait), as in the
// batch-1 kernel: one counter, thread 0 arrives with a release and polls
__device__ void bgrid_arrive(const BatchParams &p, unsigned &epoch)
{
    cta_sync();
    epoch += 1;
    if (threadIdx.x == 0) red_release_gpu(p.bar, 1u);
}
__device__ bool bgrid_wait(BSmem *sm, const BatchParams &p, unsigned epoch, int &bci)
{
    if (threadIdx.x == 0) {
        const unsigned target = epoch * gridDim.x;
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
    }
    cta_sync();
    const bool ok = ld_vol(&sm->bc[bci]) != 0;
    bci ^= 1;
    return ok;
}
// thread 0 waits (bounded) for a staging barrier; the CTA adopts its verdict
__device__ bool bstage_wait(BSmem *sm, const BatchParams &p, uint64_t *bar, uint32_t &par, int &bci)
{
    if (threadIdx.x == 0) {
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
    }
    cta_sync();
    const bool ok = ld_vol(&sm->bc[bci]) != 0;
    bci ^= 1;
    if (ok) {
        mbar_test(bar, par);
        par ^= 1;
    }
    return ok;
}

template <int WF>
__global__ void __launch_bounds__(kThreads, 1) batch_kernel(const __grid_constant__ BatchParams p)
{
    extern __shared__ __align__(1024) uint8_t dyn[];
    __shared__ BSmem sm;
    uint8_t *const xs = dyn;                       // [kNB][d] x (hi), 16-bit, chunk-permuted
    uint8_t *const stg = dyn + kXBytes;            // staging
    float *const gred = reinterpret_cast<float *>(dyn + kXBytes + kBStage);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.x, S = gridDim.x;
    const int d = p.d, r = p.r, nb = p.nb;
    // 16-bit parts of x and h in the gate/up/down products (columns part * TPL + token)
    constexpr int NPX = WF == kBF16 ? 2 : 1;
    constexpr int TPL = kNB / NPX;                 // tokens per launch at most
    const int s0 = p.strip_off[b], ns = p.strip_off[b + 1] - s0;
    const int c0 = 8 * p.grp_off[b], ncol = 8 * (p.grp_off[b + 1] - p.grp_off[b]);
    const int a0 = int((long long)b * r / S), a1 = int((long long)(b + 1) * r / S);
    const int l0 = p.layer_begin, l1 = p.layer_end;
    const int nks_d = d / 16;                      // 16-column steps of a row of d
    const int g = lane >> 2, tq = lane & 3;
    constexpr int kParts = WF == kBF16 ? 3 : 2;   // 16-bit parts of t (22 / 24 significant bits)
    const int tstride = r + 8;                     // t-part row (one column of the B operand), elements
    uint16_t *const tpart = reinterpret_cast<uint16_t *>(stg);
    // V rows of t per round (row stride vrow + 16 bytes, so the rows of a
    // matrix load fall in different bank groups), after the x remainders
    const int vstride = p.vrow + 16;
    const int vcap = min(16, (kBStage - kXBytes) / vstride);
    // U rows per logit round (a multiple of 8), after the t parts
    const int ucap = max(8, min(kMaxStrip, (kBStage - kTPartBytes) / p.urow) & ~7);
    // gather slots: gate | up | down rows of one neuron, 128-byte aligned,
    // shifted by 16 bytes per slot (bank groups of the matrix loads)
    const int slot_bytes = (p.gu_bytes + p.wrow + 127) & ~127;
    const int gu_rows = p.gated ? 2 : 1;

    unsigned epoch = 0;
    int bci = 0;
    uint32_t par_v = 0, par_u = 0, par_g = 0;
    bool pend_v = false, pend_u = false, pend_g = false;

    if (tid == 0) {
        mbar_init(&sm.bar_v, 1);
        mbar_init(&sm.bar_u, 1);
        mbar_init(&sm.bar_g, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // x rows of absent tokens stay zero
    for (int i = tid; i < kNB * d / 8; i += kThreads)
        if ((i / (d / 8)) % TPL >= nb) reinterpret_cast<uint4 *>(xs)[i] = make_uint4(0u, 0u, 0u, 0u);
    cta_sync();

    // ---------------- column phase: this CTA's columns of every token -------
    // li_in: index (in the launch) of the layer whose input r is formed here
    auto column_phase = [&](int li_in, bool from_partials) {
        const int nq = ncol / 4;
        for (int task = warp; task < nb * nq; task += kConsumerWarps) {
            const int t = task / nq, qq = task % nq;
            const int q = c0 / 4 + qq;
            float4 rv = __ldcg(reinterpret_cast<const float4 *>(p.resid + size_t(t) * d) + q);
            if (from_partials) {
                float4 sacc = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int c = lane; c < S; c += 32) {
                    const float4 v = __ldcg(reinterpret_cast<const float4 *>(p.partials + (size_t(c) * nb + t) * d) + q);
                    sacc.x += v.x; sacc.y += v.y; sacc.z += v.z; sacc.w += v.w;
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    sacc.x += __shfl_xor_sync(0xffffffffu, sacc.x, o);
                    sacc.y += __shfl_xor_sync(0xffffffffu, sacc.y, o);
                    sacc.z += __shfl_xor_sync(0xffffffffu, sacc.z, o);
                    sacc.w += __shfl_xor_sync(0xffffffffu, sacc.w, o);
                }
                rv.x += sacc.x; rv.y += sacc.y; rv.z += sacc.z; rv.w += sacc.w;
                if (lane == 0) __stcg(reinterpret_cast<float4 *>(p.resid + size_t(t) * d) + q, rv);
            }
            if (lane == 0) *reinterpret_cast<float4 *>(&sm.rsl[t][4 * qq]) = rv;
        }
        cta_sync();
        if (p.trace && li_in < l1 - l0)
            for (int i = tid; i < nb * ncol; i += kThreads) {
                const int t = i / ncol, j = i % ncol;
                __stcg(p.trace + (size_t(li_in) * p.ntok + p.tok0 + t) * d + c0 + j, sm.rsl[t][j]);
            }
        // per-CTA sums of squares, one warp per token (fixed order)
        if (warp < nb) {
            float s = 0.f;
            for (int j = lane; j < ncol; j += 32) s = fmaf(sm.rsl[warp][j], sm.rsl[warp][j], s);
            s = warp_sum(s);
            if (lane == 0) __stcg(p.ss + size_t(b) * kNB + warp, s);
        }
    };

    column_phase(0, false);
    bgrid_arrive(p, epoch);
    bool ok = bgrid_wait(&sm, p, epoch, bci);

    for (int l = l0; ok && l < l1; ++l) {
        const int li = l - l0;
        const ExpertDev ex = p.ex[l];
        const uint8_t *vrm = p.vrm[l];
        // ---------------- [A] x of every token, rows [a0, a1) of t ------------
        // the first round of this CTA's V rows starts moving at once
        const int nv0 = min(vcap, a1 - a0);
        if (tid == 0 && nv0 > 0) {
            mbar_arrive_tx(&sm.bar_v, uint32_t(nv0) * p.vrow);
            for (int i = 0; i < nv0; ++i)
                bulk_g2s(stg + kXBytes + size_t(i) * vstride, vrm + size_t(a0 + i) * p.vrow, uint32_t(p.vrow), &sm.bar_v);
        }
        pend_v = nv0 > 0;
        if (tid < nb) {
            float s = 0.f;
            for (int c = 0; c < S; ++c) s += __ldcg(p.ss + size_t(c) * kNB + tid);
            sm.inv[tid] = 1.f / sqrtf(s / float(d) + p.eps);
        }
        for (int i = tid; i < ns; i += kThreads) sm.cbuf[i] = __ldg(ex.c + s0 + i);
        cta_sync();
        // x = r * inv as hi + lo: F16 keeps lo in the staging buffer (for the
        // predictor only), BF16 in x rows TPL + t; 8 elements per step
        for (int i = tid; i < nb * d / 8; i += kThreads) {
            const int t = i / (d / 8), j = (i % (d / 8)) * 8;
            const float4 q0 = __ldcg(reinterpret_cast<const float4 *>(p.resid + size_t(t) * d + j));
            const float4 q1 = __ldcg(reinterpret_cast<const float4 *>(p.resid + size_t(t) * d + j + 4));
            const float v[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
            uint16_t hi[8], lo[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float x = v[e] * sm.inv[t];
                hi[e] = to16<WF>(x);
                lo[e] = to16<WF>(x - from16<WF>(hi[e]));
            }
            *reinterpret_cast<uint4 *>(xs + xoff(t, j, d)) = *reinterpret_cast<const uint4 *>(hi);
            if constexpr (NPX == 2) *reinterpret_cast<uint4 *>(xs + xoff(TPL + t, j, d)) = *reinterpret_cast<const uint4 *>(lo);
            else *reinterpret_cast<uint4 *>(stg + xoff(t, j, d)) = *reinterpret_cast<const uint4 *>(lo);
        }
        // absent tokens: zero remainders too
        if constexpr (NPX == 1)
            for (int i = tid; i < (kNB - nb) * d / 8; i += kThreads)
                reinterpret_cast<uint4 *>(stg + size_t(nb) * d * 2)[i] = make_uint4(0u, 0u, 0u, 0u);
        cta_sync();
        // t rows by tensor-core dots: A = 16 V rows (rows past the round's
        // last repeat its first; their results are dropped), B = x hi and lo
        for (int v0 = a0; v0 < a1 && ok; v0 += vcap) {
            const int nv = min(vcap, a1 - v0);
            if (v0 > a0) {
                if (tid == 0) {
                    mbar_arrive_tx(&sm.bar_v, uint32_t(nv) * p.vrow);
                    for (int i = 0; i < nv; ++i)
                        bulk_g2s(stg + kXBytes + size_t(i) * vstride, vrm + size_t(v0 + i) * p.vrow, uint32_t(p.vrow), &sm.bar_v);
                }
                pend_v = true;
            }
            if (!bstage_wait(&sm, p, &sm.bar_v, par_v, bci)) { ok = false; break; }
            pend_v = false;
            float c[4] = {0.f, 0.f, 0.f, 0.f};
            const int row = (lane & 15) < nv ? (lane & 15) : 0;
            const uint8_t *arow = stg + kXBytes + size_t(row) * vstride;
            const int k0 = warp * nks_d / kConsumerWarps, k1 = (warp + 1) * nks_d / kConsumerWarps;
            for (int ks = k0; ks < k1; ++ks) {
                uint32_t a[4];
                ldsm_x4(arow + (2 * ks + (lane >> 4)) * 16, a[0], a[1], a[2], a[3]);
                const int tr = lane & 7, jc = 16 * ks + ((lane >> 3) & 1) * 8;
                uint32_t bh0, bh1;
                ldsm_x2(xs + xoff(tr, jc, d), bh0, bh1);
                mma16816<WF>(c, a[0], a[1], a[2], a[3], bh0, bh1);
                if constexpr (NPX == 1) {
                    uint32_t bl0, bl1;
                    ldsm_x2(stg + xoff(tr, jc, d), bl0, bl1);
                    mma16816<WF>(c, a[0], a[1], a[2], a[3], bl0, bl1);
                }
            }
            // rows g, g + 8; tokens 2tq, 2tq + 1
            gred[(warp * 16 + g) * kNB + 2 * tq] = c[0];
            gred[(warp * 16 + g) * kNB + 2 * tq + 1] = c[1];
            gred[(warp * 16 + g + 8) * kNB + 2 * tq] = c[2];
            gred[(warp * 16 + g + 8) * kNB + 2 * tq + 1] = c[3];
            cta_sync();
            if (tid < nv * nb) {
                const int rr = tid / nb, t = tid % nb;
                float s = 0.f;
                for (int w = 0; w < kConsumerWarps; ++w) {
                    s += gred[(w * 16 + rr) * kNB + t];
                    if constexpr (NPX == 2) s += gred[(w * 16 + rr) * kNB + TPL + t];
                }
                __stcg(p.t_buf + size_t(t) * r + v0 + rr, s);
            }
            cta_sync();
        }
        if (!ok) break;
        bgrid_arrive(p, epoch);
        // the first U round lands during the barrier
        const int nu0 = min(ucap, ns);
        if (tid == 0 && nu0 > 0) {
            mbar_arrive_tx(&sm.bar_u, uint32_t(nu0) * p.urow);
            stage_copy(stg + kTPartBytes, ex.U + size_t(s0) * p.urow, uint32_t(nu0) * p.urow, &sm.bar_u);
        }
        pend_u = nu0 > 0;
        if (!bgrid_wait(&sm, p, epoch, bci)) { ok = false; break; }

        // ---------------- [B] z = U t - c, token masks, union ---------------
        // t parts: column n = part * 8 + token, tstride elements per column
        for (int i = tid; i < kNB * r; i += kThreads) {
            const int t = i / r, k = i % r;
            const float tv = t < nb ? __ldcg(p.t_buf + size_t(t) * r + k) : 0.f;
            if constexpr (WF == kBF16) {
                const __nv_bfloat16 h0 = __float2bfloat16_rn(tv);
                const float r1 = tv - __bfloat162float(h0);
                const __nv_bfloat16 h1 = __float2bfloat16_rn(r1);
                tpart[size_t(t) * tstride + k] = __bfloat16_as_ushort(h0);
                tpart[size_t(8 + t) * tstride + k] = __bfloat16_as_ushort(h1);
                tpart[size_t(16 + t) * tstride + k] = __bfloat16_as_ushort(__float2bfloat16_rn(r1 - __bfloat162float(h1)));
            } else {
                const __half h0 = __float2half_rn(tv);
                tpart[size_t(t) * tstride + k] = __half_as_ushort(h0);
                tpart[size_t(8 + t) * tstride + k] = __half_as_ushort(__float2half_rn(tv - __half2float(h0)));
            }
        }
        for (int i = tid; i < ns; i += kThreads) sm.zmask[i] = 0u;
        cta_sync();
        const int nks_r = r / 16;
        for (int row0 = 0; row0 < ns && ok; row0 += ucap) {
            const int n = min(ucap, ns - row0);
            if (row0 > 0) {
                if (tid == 0) {
                    mbar_arrive_tx(&sm.bar_u, uint32_t(n) * p.urow);
                    stage_copy(stg + kTPartBytes, ex.U + size_t(s0 + row0) * p.urow, uint32_t(n) * p.urow, &sm.bar_u);
                }
                pend_u = true;
            }
            if (!bstage_wait(&sm, p, &sm.bar_u, par_u, bci)) { ok = false; break; }
            pend_u = false;
            const int nmt = (n + 15) / 16;
            const int kg = max(1, min(4, kConsumerWarps / nmt));
            if (warp < nmt * kg) {
                const int mt = warp % nmt, grp = warp / nmt;
                const int k0 = grp * nks_r / kg, k1 = (grp + 1) * nks_r / kg;
                float c[3][4];
#pragma unroll
                for (int q = 0; q < 3; ++q) c[q][0] = c[q][1] = c[q][2] = c[q][3] = 0.f;
                const int rowa = min(mt * 16 + (lane & 15), n - 1);
                const int key = p.u_swz ? (rowa & 7) : 0;
                const uint8_t *ua = stg + kTPartBytes + size_t(rowa) * p.urow;
                for (int ks = k0; ks < k1; ++ks) {
                    const int chunk = 2 * ks + (lane >> 4);
                    uint32_t a[4];
                    ldsm_x4(ua + ((chunk & ~7) | ((chunk ^ key) & 7)) * 16, a[0], a[1], a[2], a[3]);
#pragma unroll
                    for (int q = 0; q < kParts; ++q) {
                        const uint16_t *bp = tpart + size_t(q * 8 + g) * tstride + ks * 16 + 2 * tq;
                        const uint32_t b0 = *reinterpret_cast<const uint32_t *>(bp);
                        const uint32_t b1 = *reinterpret_cast<const uint32_t *>(bp + 8);
                        mma16816<WF>(c[q], a[0], a[1], a[2], a[3], b0, b1);
                    }
                }
                float z[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int q = 0; q < kParts; ++q) {
                    z[0] += c[q][0]; z[1] += c[q][1]; z[2] += c[q][2]; z[3] += c[q][3];
                }
                // zq[grp][row][token], nmt * 16 rows per group
                float *zq = gred + size_t(grp) * nmt * 16 * kNB;
                zq[(mt * 16 + g) * kNB + 2 * tq] = z[0];
                zq[(mt * 16 + g) * kNB + 2 * tq + 1] = z[1];
                zq[(mt * 16 + g + 8) * kNB + 2 * tq] = z[2];
                zq[(mt * 16 + g + 8) * kNB + 2 * tq + 1] = z[3];
            }
            cta_sync();
            for (int i = tid; i < n * nb; i += kThreads) {
                const int rr = i / nb, t = i % nb;
                float s = 0.f;
                for (int q = 0; q < kg; ++q) s += gred[(size_t(q) * nmt * 16 + rr) * kNB + t];
                const float z = s - sm.cbuf[row0 + rr];
                if (z > p.threshold) atomicOr(&sm.zmask[row0 + rr], 1u << t);
            }
            cta_sync();
        }
        if (!ok) break;
        // union of the strip in ascending order (warp 0), per-token mask bits
        if (warp == 0) {
            int cnt = 0, tot = 0;
            const int words = (p.F + 31) / 32;
            for (int base = 0; base < ns; base += 32) {
                const int loc = base + lane;
                const uint32_t m = loc < ns ? sm.zmask[loc] : 0u;
                const unsigned bal = __ballot_sync(0xffffffffu, m != 0u);
                if (m) {
                    const int pos = cnt + __popc(bal & ((1u << lane) - 1u));
                    const int gp = s0 + loc;
                    __stcg(p.pub + size_t(b) * kMaxStrip + pos,
                           (unsigned long long)(unsigned(m << 24) | unsigned(gp)) |
                               ((unsigned long long)__float_as_uint(sm.cbuf[loc]) << 32));
                    if (p.masks)
                        for (int t = 0; t < nb; ++t)
                            if ((m >> t) & 1u)
                                atomicOr(p.masks + (size_t(li) * p.ntok + p.tok0 + t) * words + (gp >> 5),
                                         1u << (gp & 31));
                    sm.lst[pos] = gp;
                }
                tot += __reduce_add_sync(0xffffffffu, __popc(m));
                cnt += __popc(bal);
            }
            if (lane == 0) {
                __stcg(p.counts + b, cnt);
                sm.lst_n = cnt;
                if (p.stats) {
                    atomicAdd(p.stats + li * 4 + 0, cnt);
                    atomicAdd(p.stats + li * 4 + 1, tot);
                }
            }
        }
        bgrid_arrive(p, epoch);
        // the union's rows start moving towards L2 once this CTA has arrived
        for (int j = tid; j < sm.lst_n; j += kThreads) {
            const int gp = sm.lst[j];
            prefetch_l2(ex.Wgu + size_t(gp) * p.rec_bytes, uint32_t(p.spec ? p.rec_bytes : p.gu_bytes));
            if (!p.spec) prefetch_l2(ex.Wd + size_t(gp) * p.wd_stride, uint32_t(p.wrow));
        }
        if (!bgrid_wait(&sm, p, epoch, bci)) { ok = false; break; }

        // ---------------- [C] balanced gather of the union -------------------
        {
            const int cnt = tid < S ? __ldcg(p.counts + tid) : 0;
            int inc = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += v;
            }
            if (lane == 31) sm.red[warp] = inc;
            cta_sync();
            if (tid <= S) {
                int pre = inc - cnt;
                for (int w = 0; w < warp; ++w) pre += sm.red[w];
                sm.scan[tid] = pre;
            }
            cta_sync();
            const int ntot = sm.scan[S];
            const int lo = int((long long)b * ntot / S), hi = int((long long)(b + 1) * ntot / S);
            for (int j = lo + tid; j < hi; j += kThreads) {
                int q0 = 0, q1 = S;
                while (q1 - q0 > 1) {
                    const int mid = (q0 + q1) >> 1;
                    if (sm.scan[mid] <= j) q0 = mid;
                    else q1 = mid;
                }
                const unsigned long long w = __ldcg(p.pub + size_t(q0) * kMaxStrip + (j - sm.scan[q0]));
                sm.glst[j - lo] = int(unsigned(w));
                sm.gc[j - lo] = __uint_as_float(unsigned(w >> 32));
            }
            if (tid == 0) {
                sm.share_n = hi - lo;
                sm.nzu = 0;
            }
            cta_sync();
        }
        const int m = sm.share_n;
        const int nmt_d = d / 256;     // 16-row tiles of y per warp
        float acc[kBD / 256][4];
#pragma unroll
        for (int i = 0; i < kBD / 256; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
        auto slot_at = [&](int n) -> uint8_t * { return stg + size_t(n) * slot_bytes + (n & 7) * 16; };
        for (int j0 = 0; j0 < m && ok; j0 += kBRound) {
            const int k = min(kBRound, m - j0);
            if (warp == 0) {
                if (lane == 0) mbar_arrive_tx(&sm.bar_g, uint32_t(k) * uint32_t(p.gu_bytes + p.wrow));
                __syncwarp();
                if (lane < k) {
                    const int pos = sm.glst[j0 + lane] & 0xffffff;
                    uint8_t *slot = slot_at(lane);
                    if (p.spec) {
                        stage_copy(slot, ex.Wgu + size_t(pos) * p.rec_bytes, uint32_t(p.rec_bytes), &sm.bar_g);
                    } else {
                        stage_copy(slot, ex.Wgu + size_t(pos) * p.rec_bytes, uint32_t(p.gu_bytes), &sm.bar_g);
                        stage_copy(slot + p.gu_bytes, ex.Wd + size_t(pos) * p.wd_stride, uint32_t(p.wrow), &sm.bar_g);
                    }
                }
            }
            pend_g = true;
            if (!bstage_wait(&sm, p, &sm.bar_g, par_g, bci)) { ok = false; break; }
            pend_g = false;
            // G = W_gu (16 slots x d) X^T (d x 8 tokens), K split over the warps
            {
                float cg[4] = {0.f, 0.f, 0.f, 0.f}, cu[4] = {0.f, 0.f, 0.f, 0.f};
                const int sl = (lane & 15) < k ? (lane & 15) : 0;
                const uint8_t *ga = slot_at(sl);
                const int k0 = warp * nks_d / kConsumerWarps, k1 = (warp + 1) * nks_d / kConsumerWarps;
                for (int ks = k0; ks < k1; ++ks) {
                    const int tr = lane & 7, jc = 16 * ks + ((lane >> 3) & 1) * 8;
                    uint32_t b0, b1;
                    ldsm_x2(xs + xoff(tr, jc, d), b0, b1);
                    uint32_t a[4];
                    ldsm_x4(ga + (2 * ks + (lane >> 4)) * 16, a[0], a[1], a[2], a[3]);
                    mma16816<WF>(cg, a[0], a[1], a[2], a[3], b0, b1);
                    if (gu_rows == 2) {
                        ldsm_x4(ga + p.wrow + (2 * ks + (lane >> 4)) * 16, a[0], a[1], a[2], a[3]);
                        mma16816<WF>(cu, a[0], a[1], a[2], a[3], b0, b1);
                    }
                }
                // gred[warp][slot][token][gate, up]
                float *gw = gred + size_t(warp) * 16 * kNB * 2;
                gw[(g * kNB + 2 * tq) * 2] = cg[0];
                gw[(g * kNB + 2 * tq + 1) * 2] = cg[1];
                gw[((g + 8) * kNB + 2 * tq) * 2] = cg[2];
                gw[((g + 8) * kNB + 2 * tq + 1) * 2] = cg[3];
                gw[(g * kNB + 2 * tq) * 2 + 1] = cu[0];
                gw[(g * kNB + 2 * tq + 1) * 2 + 1] = cu[1];
                gw[((g + 8) * kNB + 2 * tq) * 2 + 1] = cu[2];
                gw[((g + 8) * kNB + 2 * tq + 1) * 2 + 1] = cu[3];
            }
            cta_sync();
            // h of (slot, token): fixed-order sum over the warps, the token's own mask
            if (tid < 16 * kNB) {
                const int sl = tid / kNB, t = tid % kNB;
                float h = 0.f;
                if (sl < k && t < nb && ((unsigned(sm.glst[j0 + sl]) >> (24 + t)) & 1u)) {
                    float gs = 0.f, us = 0.f;
                    for (int w = 0; w < kConsumerWarps; ++w) {
#pragma unroll
                        for (int q = 0; q < NPX; ++q) {
                            gs += gred[((size_t(w) * 16 + sl) * kNB + q * TPL + t) * 2];
                            us += gred[((size_t(w) * 16 + sl) * kNB + q * TPL + t) * 2 + 1];
                        }
                    }
                    h = act_h(p.act, gs - sm.gc[j0 + sl], us);
                }
                // (slot, t) for t < TPL writes h's parts: column t, and column TPL + t (BF16)
                if (t < TPL) {
                    const uint16_t hh = to16<WF>(h);
                    sm.hs[t][sl] = hh;
                    if constexpr (NPX == 2) sm.hs[TPL + t][sl] = to16<WF>(h - from16<WF>(hh));
                }
                // a union neuron whose h is non-zero for some token
                const unsigned nzb = __ballot_sync(0xffffffffu, h != 0.f);
                if (lane % kNB == 0 && ((nzb >> lane) & 0xffu)) atomicAdd(&sm.nzu, 1);
            }
            cta_sync();
            // Y^T += W_d^T (d x 16 slots) H (16 slots x 8 tokens): this warp's rows
            {
                const int sl = (lane & 7) + ((lane >> 4) << 3);
                const uint8_t *da = slot_at(sl < k ? sl : 0) + p.gu_bytes;
                const int dofs = ((lane >> 3) & 1) * 8;
                const uint32_t b0 = *reinterpret_cast<const uint32_t *>(&sm.hs[g][2 * tq]);
                const uint32_t b1 = *reinterpret_cast<const uint32_t *>(&sm.hs[g][2 * tq + 8]);
#pragma unroll
                for (int i = 0; i < kBD / 256; ++i) {
                    if (i < nmt_d) {
                        const int m0 = (warp * nmt_d + i) * 16;
                        uint32_t a[4];
                        ldsm_x4_t(da + (m0 + dofs) * 2, a[0], a[1], a[2], a[3]);
                        mma16816<WF>(acc[i], a[0], a[1], a[2], a[3], b0, b1);
                    }
                }
            }
            cta_sync();   // the staging buffer and hs are reused by the next round
        }
        if (!ok) break;
        if (tid == 0 && p.stats) atomicAdd(p.stats + li * 4 + 2, sm.nzu);
        // per-CTA partial of y for every token: rows g, g + 8 of each tile,
        // columns 2tq, 2tq + 1 (BF16: the parts of token j sit in columns j and
        // TPL + j, i.e. lanes tq and tq + 2: summed into the lower lane)
#pragma unroll
        for (int i = 0; i < kBD / 256; ++i) {
            if constexpr (NPX == 2) {
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[i][q] += __shfl_down_sync(0xffffffffu, acc[i][q], 2);
            }
            if (i < nmt_d && (NPX == 1 || tq < 2)) {
                const int m0 = (warp * nmt_d + i) * 16;
                const int t0 = 2 * tq, t1 = 2 * tq + 1;
                if (t0 < nb) {
                    __stcg(p.partials + (size_t(b) * nb + t0) * d + m0 + g, acc[i][0]);
                    __stcg(p.partials + (size_t(b) * nb + t0) * d + m0 + g + 8, acc[i][2]);
                }
                if (t1 < nb) {
                    __stcg(p.partials + (size_t(b) * nb + t1) * d + m0 + g, acc[i][1]);
                    __stcg(p.partials + (size_t(b) * nb + t1) * d + m0 + g + 8, acc[i][3]);
                }
            }
        }
        bgrid_arrive(p, epoch);
        if (!bgrid_wait(&sm, p, epoch, bci)) { ok = false; break; }
        // ---------------- column phase: r of the next layer -------------------
        column_phase(li + 1, true);
        bgrid_arrive(p, epoch);
        if (!bgrid_wait(&sm, p, epoch, bci)) { ok = false; break; }
    }
    // an early exit may leave copies in flight: let them land (bounded)
    if (tid == 0) {
        const long long t0 = gtimer();
        if (pend_v) while (!mbar_test(&sm.bar_v, par_v) && gtimer() - t0 < p.wait_ns) {}
        if (pend_u) while (!mbar_test(&sm.bar_u, par_u) && gtimer() - t0 < p.wait_ns) {}
        if (pend_g) while (!mbar_test(&sm.bar_g, par_g) && gtimer() - t0 < p.wait_ns) {}
    }
}

}  // namespace

int batch_max_tokens() { return kNB; }
int batch_tokens_per_launch(int wfmt) { return wfmt == kBF16 ? kNB / 2 : kNB; }
int batch_max_d() { return kBD; }

cudaError_t launch_batch(int wfmt, const BatchLaunch &L, cudaStream_t st)
{
    BatchParams p{};
    p.ex = L.ex;
    p.vrm = L.vrm;
    p.strip_off = L.strip_off;
    p.grp_off = L.grp_off;
    p.d = L.d; p.F = L.F; p.r = L.r; p.act = L.act; p.gated = L.gated; p.S = L.S; p.nb = L.nb;
    p.layer_begin = L.layer_begin; p.layer_end = L.layer_end;
    p.threshold = L.threshold; p.eps = L.eps;
    p.vrow = L.vrow; p.urow = L.urow; p.wrow = L.wrow; p.gu_bytes = L.gu_bytes; p.rec_bytes = L.rec_bytes;
    p.wd_stride = L.wd_stride; p.spec = L.spec; p.u_swz = L.u_swz;
    p.resid = L.resid; p.trace = L.trace; p.stats = L.stats; p.masks = L.masks;
    p.ntok = L.ntok; p.tok0 = L.tok0;
    p.t_buf = L.t_buf; p.ss = L.ss; p.partials = L.partials; p.counts = L.counts; p.pub = L.pub;
    p.bar = L.bar; p.err = L.err; p.wait_ns = L.wait_ns;
    void *fn = wfmt == kBF16 ? (void *)batch_kernel<kBF16> : (void *)batch_kernel<kF16>;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kBSmem);
    if (e != cudaSuccess) return e;
    void *args[] = {&p};
    return cudaLaunchCooperativeKernel(fn, dim3(p.S), dim3(kThreads), args, kBSmem, st);
}

int batch_max_blocks_per_sm(int wfmt)
{
    void *fn = wfmt == kBF16 ? (void *)batch_kernel<kBF16> : (void *)batch_kernel<kF16>;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kBSmem) != cudaSuccess) return 0;
    int blocks = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, fn, kThreads, kBSmem) != cudaSuccess) return 0;
    return blocks;
}

}  // namespace pi
