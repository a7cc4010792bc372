// pi_host.cu -- host side of the C ABI declared in include/pi_ffn.h.
//
// Validates every call before enqueuing work, owns the per-layer device
// memory (weights in neuron-table order) and the per-handle scratch, builds
// the neuron tables, and launches the decode kernel (pi_decode.cu) and the
// prefill kernels (pi_prefill.cu).
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>
#include <numeric>
#include <vector>

#include "../../include/pi_ffn.h"
#include "pi_internal.h"
#include "pi_prefill.h"

namespace {

thread_local char g_msg[512] = "no error";

pi_status fail(pi_status st, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof g_msg, fmt, ap);
    va_end(ap);
    return st;
}

pi_status cuda_fail(cudaError_t e, const char *what)
{
    return fail(e == cudaErrorMemoryAllocation ? PI_ERR_OOM : PI_ERR_CUDA, "%s: %s (%s)", what,
                cudaGetErrorName(e), cudaGetErrorString(e));
}

#define PI_CUDA(call, what)                                   \
    do {                                                      \
        cudaError_t e_ = (call);                              \
        if (e_ != cudaSuccess) return cuda_fail(e_, what);    \
    } while (0)

int fmt_of(pi_dtype t)
{
    switch (t) {
    case PI_F32: return pi::kF32;
    case PI_F16: return pi::kF16;
    case PI_BF16: return pi::kBF16;
    case PI_INT4G32: return pi::kI4;
    case PI_I8: return pi::kI8;
    }
    return -1;
}

int elem_bytes(pi_dtype t) { return t == PI_F32 ? 4 : (t == PI_I8 ? 1 : 2); }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

void pi::set_last_error(const char *msg)
{
    snprintf(g_msg, sizeof g_msg, "%s", msg);
}

struct pi_ffn {
    pi_ffn_desc desc{};
    int S = 0;                       // strips = CTAs of the decode kernel
    int wfmt = 0, pfmt = 0, gated = 0;
    int vrow = 0, urow = 0, wrow = 0;
    int u_swz = 0;
    bool spec = false;
    std::vector<int32_t> strip_off;
    std::vector<int32_t> grp_off;              // column slices in 8-column groups
    std::vector<std::vector<int32_t>> perm;   // [layer * E + e]
    std::vector<uint8_t *> mem;               // [layer * E + e]
    std::vector<uint8_t *> router_mem;        // [layer]
    std::vector<char> loaded;                 // [layer]
    std::vector<pi::ExpertDev> h_ex;          // [layer * E]
    pi::ExpertDev *d_ex = nullptr;
    const uint8_t **d_router = nullptr;
    int32_t *d_strip_off = nullptr;
    int32_t *d_grp_off = nullptr;
    // scratch
    uint8_t *scratch = nullptr;
    float *io = nullptr;
    unsigned long long *yfix = nullptr;       // [2 d] each layer's y in fixed point, by layer parity
    float *rbuf = nullptr;                    // [2 d] each layer's input, by layer parity
    int32_t *lists = nullptr, *counts = nullptr;
    unsigned long long *pub = nullptr;
    unsigned *bar = nullptr;
    int *err = nullptr;
    long long wait_ns = 2000000000LL;
    int debug_flags = 0;
    long long *prof = nullptr;
    pi::PrefillState *prefill = nullptr;
    // small-batch decode: workspace and a table of the layers' V, made on first use
    uint8_t *bscratch = nullptr;
    std::vector<char> vrm_ok;                 // [layer] the V table's entry is current
    const uint8_t **d_vrm = nullptr;          // [layer] each layer's V rows
    int batch_fits = -1;                      // batch kernel co-resident with S CTAs (-1 unknown)
    int hot_k = 0;                            // records kept in HBM per strip (0 = all)
    std::vector<uint8_t *> host_mem;          // [layer * E + e] pinned cold records
};

extern "C" {

const char *pi_last_error(void) { return g_msg; }

pi_status pi_ffn_create(const pi_ffn_desc *desc, pi_ffn_t *out)
{
    if (!desc || !out) return fail(PI_ERR_INVALID_ARG, "pi_ffn_create: null argument");
    *out = nullptr;
    const pi_ffn_desc &D = *desc;
    if (D.n_layers < 1) return fail(PI_ERR_INVALID_ARG, "n_layers must be >= 1");
    if (D.d_model < 256 || D.d_model % 256 != 0 || D.d_model > 8192)
        return fail(PI_ERR_INVALID_ARG, "d_model must be a multiple of 256 in [256, 8192]");
    if (D.w_dtype == PI_F32 && D.d_model > 4096)
        return fail(PI_ERR_UNSUPPORTED, "F32 weights need d_model <= 4096");
    if (D.d_ff < 1) return fail(PI_ERR_INVALID_ARG, "d_ff must be >= 1");
    if (D.act < PI_ACT_RELU || D.act > PI_ACT_DRELU) return fail(PI_ERR_INVALID_ARG, "bad act");
    if (fmt_of(D.w_dtype) < 0 || D.w_dtype == PI_I8) return fail(PI_ERR_INVALID_ARG, "bad w_dtype");
    if (fmt_of(D.pred_dtype) < 0 || D.pred_dtype == PI_INT4G32)
        return fail(PI_ERR_INVALID_ARG, "pred_dtype must be F32, F16, BF16 or I8");
    const bool pair_ok = (D.w_dtype == PI_F32 && D.pred_dtype == PI_F32) ||
                         (D.w_dtype == PI_F16 && (D.pred_dtype == PI_F16 || D.pred_dtype == PI_I8)) ||
                         (D.w_dtype == PI_BF16 && (D.pred_dtype == PI_BF16 || D.pred_dtype == PI_I8)) ||
                         (D.w_dtype == PI_INT4G32 && D.pred_dtype != PI_F32);
    if (!pair_ok)
        return fail(PI_ERR_UNSUPPORTED,
                    "supported (w_dtype, pred_dtype): (F32,F32) (F16,F16) (BF16,BF16) (F16,I8) (BF16,I8) "
                    "(INT4G32,F16) (INT4G32,BF16) (INT4G32,I8)");
    const int pb = elem_bytes(D.pred_dtype);
    const int max_rank = D.pred_dtype == PI_F32 ? 512 : 1024;
    if (D.rank < 1 || D.rank % 16 != 0 || D.rank > max_rank)
        return fail(PI_ERR_INVALID_ARG, "rank must be a multiple of 16 and <= %d", max_rank);
    if (D.pred_dtype == PI_I8 && D.rank % 32 != 0)
        return fail(PI_ERR_INVALID_ARG, "an I8 predictor needs rank a multiple of 32");
    if (D.n_experts == 1) {
        if (D.top_k != 1) return fail(PI_ERR_INVALID_ARG, "a dense FFN needs top_k = 1");
    } else if (D.n_experts >= 2 && D.n_experts <= pi::kMaxExperts) {
        if (D.top_k != 2) return fail(PI_ERR_UNSUPPORTED, "MoE supports top_k = 2");
    } else {
        return fail(PI_ERR_INVALID_ARG, "n_experts must be in [1, %d]", pi::kMaxExperts);
    }
    if (D.n_experts > 1 && D.pred_dtype == PI_F32)
        return fail(PI_ERR_UNSUPPORTED, "MoE needs an F16 or BF16 predictor");
    if (D.top_k * D.rank > pi::kMaxRankTotal)
        return fail(PI_ERR_INVALID_ARG, "top_k * rank must be <= %d", pi::kMaxRankTotal);
    if (!(D.eps > 0.f) || !std::isfinite(D.threshold))
        return fail(PI_ERR_INVALID_ARG, "eps must be > 0 and threshold finite");

    int ndev = 0;
    PI_CUDA(cudaGetDeviceCount(&ndev), "cudaGetDeviceCount");
    if (D.device < 0 || D.device >= ndev) return fail(PI_ERR_INVALID_ARG, "bad device %d", D.device);
    PI_CUDA(cudaSetDevice(D.device), "cudaSetDevice");
    cudaDeviceProp prop;
    PI_CUDA(cudaGetDeviceProperties(&prop, D.device), "cudaGetDeviceProperties");
    if (prop.major != 10)
        return fail(PI_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a",
                    D.device, prop.major, prop.minor);

    pi_ffn *h = new (std::nothrow) pi_ffn;
    if (!h) return fail(PI_ERR_OOM, "host allocation failed");
    h->desc = D;
    h->wfmt = fmt_of(D.w_dtype);
    h->pfmt = fmt_of(D.pred_dtype);
    h->gated = D.act != PI_ACT_RELU;
    // ReLU / ReGLU: z > 0 nearly always means h != 0, so a predicted neuron's
    // W_down row is fetched with its input rows (speculatively)
    h->spec = D.act != PI_ACT_DRELU;
    h->vrow = D.d_model * pb;
    h->urow = D.rank * pb;
    // 16-bit predictors feed tensor-core dots through 8-row matrix loads; rows
    // of whole 128-byte groups are stored chunk-permuted so those loads do not
    // collide in shared-memory banks
    h->u_swz = D.pred_dtype != PI_F32 && h->urow % 128 == 0;
    h->wrow = D.w_dtype == PI_INT4G32 ? D.d_model / 2 + D.d_model / 16
                                      : D.d_model * elem_bytes(D.w_dtype);
    h->S = D.n_strips > 0 ? D.n_strips : prop.multiProcessorCount;

    if (h->S > pi::kMaxStrips) {
        delete h;
        return fail(PI_ERR_UNSUPPORTED, "n_strips %d exceeds %d", h->S, pi::kMaxStrips);
    }
    const int per_sm = pi::decode_max_blocks_per_sm(h->wfmt, h->pfmt, D.d_model);
    if (per_sm < 1 || h->S > per_sm * prop.multiProcessorCount) {
        delete h;
        return fail(PI_ERR_UNSUPPORTED, "n_strips %d exceeds co-resident CTAs (%d per SM x %d SMs)",
                    h->S, per_sm, prop.multiProcessorCount);
    }
    if (D.d_ff > pi::kMaxStrip * h->S) {
        delete h;
        return fail(PI_ERR_UNSUPPORTED, "d_ff %d exceeds %d neurons per strip x %d strips", D.d_ff,
                    pi::kMaxStrip, h->S);
    }
    {
        const int ng = D.d_model / 8;
        h->grp_off.resize(h->S + 1);
        for (int b = 0; b <= h->S; ++b) h->grp_off[b] = int((long long)b * ng / h->S);
        if ((ng + h->S - 1) / h->S * 8 > pi::kMaxSliceCols) {
            delete h;
            return fail(PI_ERR_UNSUPPORTED, "d_model / n_strips exceeds %d columns per strip",
                        pi::kMaxSliceCols);
        }
    }
    h->strip_off.resize(h->S + 1);
    {
        const int q = D.d_ff / h->S, rem = D.d_ff % h->S;
        h->strip_off[0] = 0;
        for (int b = 0; b < h->S; ++b) h->strip_off[b + 1] = h->strip_off[b] + q + (b < rem ? 1 : 0);
    }
    const int L = D.n_layers, E = D.n_experts;
    h->perm.assign(size_t(L) * E, {});
    h->mem.assign(size_t(L) * E, nullptr);
    h->host_mem.assign(size_t(L) * E, nullptr);
    h->router_mem.assign(L, nullptr);
    h->loaded.assign(L, 0);
    h->h_ex.assign(size_t(L) * E, pi::ExpertDev{});

    // scratch: yfix [2d] | rbuf [2d] | io [d] | lists [S kMaxStrip] | counts [S] | pub | bar | err
    // (the rows of t travel in the zeroed barrier area)
    const size_t o_yfix = 0;
    const size_t o_rbuf = up256(o_yfix + sizeof(unsigned long long) * 2 * D.d_model);
    const size_t o_io = up256(o_rbuf + sizeof(float) * 2 * D.d_model);
    const size_t o_lists = up256(o_io + sizeof(float) * D.d_model);
    const size_t o_counts = up256(o_lists + sizeof(int32_t) * size_t(h->S) * pi::kMaxStrip);
    const size_t o_pub = up256(o_counts + sizeof(int32_t) * h->S);
    const size_t o_bar = up256(o_pub + sizeof(unsigned long long) * size_t(h->S) * pi::kMaxTopK * pi::kMaxStrip);
    const size_t o_err = up256(o_bar + sizeof(unsigned) * pi::kBarWords);
    const size_t total = o_err + 256;
    cudaError_t e = cudaMalloc(&h->scratch, total);
    if (e == cudaSuccess) e = cudaMemset(h->scratch, 0, total);
    if (e == cudaSuccess) e = cudaMalloc(&h->d_ex, sizeof(pi::ExpertDev) * size_t(L) * E);
    if (e == cudaSuccess) e = cudaMemset(h->d_ex, 0, sizeof(pi::ExpertDev) * size_t(L) * E);
    if (e == cudaSuccess) e = cudaMalloc(&h->d_router, sizeof(uint8_t *) * size_t(L));
    if (e == cudaSuccess) e = cudaMemset(h->d_router, 0, sizeof(uint8_t *) * size_t(L));
    if (e == cudaSuccess) e = cudaMalloc(&h->d_grp_off, sizeof(int32_t) * (h->S + 1));
    if (e == cudaSuccess)
        e = cudaMemcpy(h->d_grp_off, h->grp_off.data(), sizeof(int32_t) * (h->S + 1), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMalloc(&h->d_strip_off, sizeof(int32_t) * (h->S + 1));
    if (e == cudaSuccess)
        e = cudaMemcpy(h->d_strip_off, h->strip_off.data(), sizeof(int32_t) * (h->S + 1),
                       cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
        pi_status st = cuda_fail(e, "pi_ffn_create: device allocation");
        pi_ffn_destroy(h);
        return st;
    }
    h->yfix = reinterpret_cast<unsigned long long *>(h->scratch + o_yfix);
    h->rbuf = reinterpret_cast<float *>(h->scratch + o_rbuf);
    h->io = reinterpret_cast<float *>(h->scratch + o_io);
    h->lists = reinterpret_cast<int32_t *>(h->scratch + o_lists);
    h->counts = reinterpret_cast<int32_t *>(h->scratch + o_counts);
    h->pub = reinterpret_cast<unsigned long long *>(h->scratch + o_pub);
    h->bar = reinterpret_cast<unsigned *>(h->scratch + o_bar);
    h->err = reinterpret_cast<int *>(h->scratch + o_err);
    *out = h;
    return PI_OK;
}

void pi_ffn_destroy(pi_ffn_t h)
{
    if (!h) return;
    cudaSetDevice(h->desc.device);
    for (uint8_t *p : h->mem) cudaFree(p);
    for (uint8_t *p : h->host_mem) cudaFreeHost(p);
    for (uint8_t *p : h->router_mem) cudaFree(p);
    cudaFree(h->d_ex);
    cudaFree(h->d_router);
    cudaFree(h->d_strip_off);
    cudaFree(h->d_grp_off);
    cudaFree(h->scratch);
    cudaFree(h->bscratch);
    cudaFree(h->d_vrm);
    pi::prefill_destroy(h->prefill);
    delete h;
}

pi_status pi_strip_offsets(pi_ffn_t h, int32_t *off_host, int *n_strips_out)
{
    if (!h) return fail(PI_ERR_INVALID_ARG, "null handle");
    if (off_host) std::memcpy(off_host, h->strip_off.data(), sizeof(int32_t) * (h->S + 1));
    if (n_strips_out) *n_strips_out = h->S;
    return PI_OK;
}

// Neuron table: rank by descending frequency (ties: lower index first), deal
// to the strips in snake order, each strip keeping its neurons hottest first.
static void build_table(const float *freq, int F, const std::vector<int32_t> &off,
                        std::vector<int32_t> &perm)
{
    perm.resize(F);
    if (!freq) {
        std::iota(perm.begin(), perm.end(), 0);
        return;
    }
    std::vector<int32_t> order(F);
    std::iota(order.begin(), order.end(), 0);
    std::sort(order.begin(), order.end(), [&](int32_t a, int32_t b) {
        if (freq[a] != freq[b]) return freq[a] > freq[b];
        return a < b;
    });
    const int S = int(off.size()) - 1;
    std::vector<int> fill(S, 0);
    int next = 0;
    for (int round = 0; next < F; ++round) {
        for (int k = 0; k < S && next < F; ++k) {
            const int b = (round & 1) ? S - 1 - k : k;
            if (fill[b] < off[b + 1] - off[b]) perm[off[b] + fill[b]++] = order[next++];
        }
    }
}

pi_status pi_ffn_load_layer(pi_ffn_t h, int layer, const pi_expert_weights *experts,
                            const void *router_dev, const float *freq_host, void *stream)
{
    if (!h || !experts) return fail(PI_ERR_INVALID_ARG, "pi_ffn_load_layer: null argument");
    const pi_ffn_desc &D = h->desc;
    if (layer < 0 || layer >= D.n_layers)
        return fail(PI_ERR_INVALID_ARG, "layer %d out of range [0, %d)", layer, D.n_layers);
    const int E = D.n_experts, F = D.d_ff, d = D.d_model, r = D.rank;
    const bool int4 = D.w_dtype == PI_INT4G32;
    for (int e = 0; e < E; ++e) {
        const pi_expert_weights &w = experts[e];
        if (!w.w_gate || !w.w_down || !w.bias || !w.U || !w.V)
            return fail(PI_ERR_INVALID_ARG, "expert %d: w_gate, w_down, bias, U and V are required", e);
        if (h->gated && !w.w_up) return fail(PI_ERR_INVALID_ARG, "expert %d: gated FFN needs w_up", e);
        if (!h->gated && w.w_up) return fail(PI_ERR_INVALID_ARG, "expert %d: non-gated FFN takes no w_up", e);
        if (int4 && (!w.s_gate || !w.s_down || (h->gated && !w.s_up)))
            return fail(PI_ERR_INVALID_ARG, "expert %d: INT4 weights need scales", e);
        if (D.pred_dtype == PI_I8 && (!w.s_U || !w.s_V))
            return fail(PI_ERR_INVALID_ARG, "expert %d: an I8 predictor needs s_U and s_V", e);
        const void *ptrs[] = {w.w_gate, w.w_up, w.w_down, w.s_gate, w.s_up, w.s_down, w.U, w.V, w.s_U, w.s_V};
        for (const void *q : ptrs)
            if (q && !aligned16(q))
                return fail(PI_ERR_INVALID_ARG, "expert %d: weight pointers must be 16-byte aligned", e);
    }
    if (E > 1 && !router_dev) return fail(PI_ERR_INVALID_ARG, "MoE layer needs a router");
    if (E == 1 && router_dev) return fail(PI_ERR_INVALID_ARG, "dense FFN takes no router");
    if (freq_host)
        for (size_t i = 0; i < size_t(E) * F; ++i)
            if (!std::isfinite(freq_host[i]))
                return fail(PI_ERR_INVALID_ARG, "freq[%zu] is not finite", i);

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    PI_CUDA(cudaSetDevice(D.device), "cudaSetDevice");
    // neuron records: gate row (+ up row); for the speculative kinds the W_down
    // row joins the record, so one copy fetches everything a neuron needs
    const int gu_bytes = (h->gated ? 2 : 1) * h->wrow;
    const bool spec = h->spec;
    const int rec_bytes = gu_bytes + (spec ? h->wrow : 0);
    // with a VRAM budget the layer memory keeps S * hot_k records (and down
    // rows); the rest go to pinned host memory (see pi_ffn_set_hot_neurons)
    const int hk = h->hot_k;
    const size_t n_dev = hk ? size_t(h->S) * hk : size_t(F);
    const size_t n_host = size_t(F) - n_dev;
    const size_t o_V = 0;
    const size_t o_U = up256(o_V + size_t(r) * h->vrow);
    const size_t o_c = up256(o_U + size_t(F) * h->urow);
    const size_t o_g = up256(o_c + sizeof(float) * F);
    const size_t o_d = up256(o_g + n_dev * rec_bytes);
    const size_t o_s = spec ? o_d : up256(o_d + n_dev * h->wrow);   // I8 predictor scales
    const bool i8 = D.pred_dtype == PI_I8;
    const size_t o_sV = up256(o_s + (i8 ? sizeof(float) * F : 0));
    const size_t total = i8 ? up256(o_sV + sizeof(float) * r) : o_s;
    int32_t *d_perm = nullptr;
    PI_CUDA(cudaMallocAsync(&d_perm, sizeof(int32_t) * F, st), "cudaMallocAsync(perm)");
    // every record (and down row) in table order, split afterwards when budgeted
    uint8_t *full_g = nullptr, *full_d = nullptr;
    if (hk) {
        PI_CUDA(cudaMallocAsync(&full_g, size_t(F) * rec_bytes, st), "cudaMallocAsync(records)");
        if (!spec) PI_CUDA(cudaMallocAsync(&full_d, size_t(F) * h->wrow, st), "cudaMallocAsync(down rows)");
    }
    for (int e = 0; e < E; ++e) {
        const size_t idx = size_t(layer) * E + e;
        const pi_expert_weights &w = experts[e];
        build_table(freq_host ? freq_host + size_t(e) * F : nullptr, F, h->strip_off, h->perm[idx]);
        if (!h->mem[idx]) PI_CUDA(cudaMalloc(&h->mem[idx], total), "cudaMalloc(layer)");
        uint8_t *m = h->mem[idx];
        uint8_t *rec_dst = hk ? full_g : m + o_g;
        uint8_t *down_dst = hk ? full_d : m + o_d;
        PI_CUDA(cudaMemcpyAsync(d_perm, h->perm[idx].data(), sizeof(int32_t) * F,
                                cudaMemcpyHostToDevice, st), "copy perm");
        // V row-major: each CTA reads its rows of t
        PI_CUDA(cudaMemcpyAsync(m + o_V, w.V, size_t(r) * h->vrow, cudaMemcpyDeviceToDevice, st), "copy V");
        if (h->u_swz) {
            PI_CUDA(pi::repack_u_swizzled(m + o_U, d_perm, F, static_cast<const uint8_t *>(w.U), h->urow,
                                          h->d_strip_off, h->S, st), "repack U");
        } else {
            const uint8_t *src[1] = {static_cast<const uint8_t *>(w.U)};
            const int rb[1] = {h->urow};
            PI_CUDA(pi::repack_rows(m + o_U, d_perm, F, 1, src, rb, st), "repack U");
        }
        PI_CUDA(pi::repack_bias(w.bias, reinterpret_cast<float *>(m + o_c), d_perm, F, st), "repack c");
        if (i8) {
            PI_CUDA(pi::repack_bias(w.s_U, reinterpret_cast<float *>(m + o_s), d_perm, F, st), "repack U scales");
            PI_CUDA(cudaMemcpyAsync(m + o_sV, w.s_V, sizeof(float) * r, cudaMemcpyDeviceToDevice, st), "copy V scales");
        }
        const uint8_t *g8 = static_cast<const uint8_t *>(w.w_gate);
        const uint8_t *u8 = static_cast<const uint8_t *>(w.w_up);
        if (int4) {
            const int qb = d / 2, sb = d / 16;
            const uint8_t *sg8 = static_cast<const uint8_t *>(w.s_gate);
            const uint8_t *su8 = static_cast<const uint8_t *>(w.s_up);
            const uint8_t *qd8 = static_cast<const uint8_t *>(w.w_down);
            const uint8_t *sd8 = static_cast<const uint8_t *>(w.s_down);
            const uint8_t *src[6] = {g8, sg8, u8, su8, qd8, sd8};
            const int rb[6] = {qb, sb, qb, sb, qb, sb};
            if (spec) {
                // gate (, up), down in one record
                const uint8_t *rs[6] = {g8, sg8, h->gated ? u8 : qd8, h->gated ? su8 : sd8, qd8, sd8};
                PI_CUDA(pi::repack_rows(rec_dst, d_perm, F, h->gated ? 6 : 4, rs, rb, st), "repack records");
            } else {
                PI_CUDA(pi::repack_rows(rec_dst, d_perm, F, h->gated ? 4 : 2, src, rb, st), "repack gate/up");
                PI_CUDA(pi::repack_rows(down_dst, d_perm, F, 2, src + 4, rb + 4, st), "repack down");
            }
        } else {
            const uint8_t *src[2] = {g8, u8};
            const int rb[2] = {h->wrow, h->wrow};
            PI_CUDA(pi::repack_rows(rec_dst, d_perm, F, h->gated ? 2 : 1, src, rb, st, rec_bytes),
                    "repack gate/up");
            PI_CUDA(pi::repack_down_transpose(static_cast<const uint8_t *>(w.w_down), spec ? rec_dst + gu_bytes : down_dst,
                                              d_perm, d, F, elem_bytes(D.w_dtype), st, spec ? rec_bytes : 0),
                    "transpose down");
        }
        pi::ExpertDev &x = h->h_ex[idx];
        x.V = m + o_V;
        x.U = m + o_U;
        x.c = reinterpret_cast<const float *>(m + o_c);
        x.Wgu = m + o_g;
        x.Wd = spec ? m + o_g + gu_bytes : m + o_d;
        x.Wgu_cold = nullptr;
        x.Wd_cold = nullptr;
        if (hk) {
            // hot records to the layer memory, the rest to pinned host memory
            const size_t host_bytes = n_host * (rec_bytes + (spec ? 0 : h->wrow));
            if (!h->host_mem[idx] && host_bytes > 0)
                PI_CUDA(cudaHostAlloc(reinterpret_cast<void **>(&h->host_mem[idx]), host_bytes, cudaHostAllocMapped),
                        "cudaHostAlloc(cold records)");
            uint8_t *hdev = nullptr;
            if (host_bytes > 0)
                PI_CUDA(cudaHostGetDevicePointer(reinterpret_cast<void **>(&hdev), h->host_mem[idx], 0),
                        "cudaHostGetDevicePointer");
            PI_CUDA(pi::split_records(full_g, m + o_g, hdev, F, rec_bytes, h->d_strip_off, h->S, hk, st),
                    "split records");
            if (!spec)
                PI_CUDA(pi::split_records(full_d, m + o_d, hdev + n_host * rec_bytes, F, h->wrow, h->d_strip_off,
                                          h->S, hk, st), "split down rows");
            x.Wgu_cold = hdev;
            x.Wd_cold = spec ? hdev + gu_bytes : hdev + n_host * rec_bytes;
        }
        x.sU = i8 ? reinterpret_cast<const float *>(m + o_s) : nullptr;
        x.sV = i8 ? reinterpret_cast<const float *>(m + o_sV) : nullptr;
        // the table is reused for the next expert: finish this one first
        PI_CUDA(cudaStreamSynchronize(st), "load_layer sync");
    }
    PI_CUDA(cudaFreeAsync(d_perm, st), "cudaFreeAsync(perm)");
    if (full_g) PI_CUDA(cudaFreeAsync(full_g, st), "cudaFreeAsync(records)");
    if (full_d) PI_CUDA(cudaFreeAsync(full_d, st), "cudaFreeAsync(down rows)");
    if (E > 1) {
        if (!h->router_mem[layer])
            PI_CUDA(cudaMalloc(&h->router_mem[layer], size_t(E) * d * 2), "cudaMalloc(router)");
        PI_CUDA(cudaMemcpyAsync(h->router_mem[layer], router_dev, size_t(E) * d * 2,
                                cudaMemcpyDeviceToDevice, st), "copy router");
        const uint8_t *rp = h->router_mem[layer];
        PI_CUDA(cudaMemcpyAsync(h->d_router + layer, &rp, sizeof(rp), cudaMemcpyHostToDevice, st),
                "router table");
    }
    PI_CUDA(cudaMemcpyAsync(h->d_ex + size_t(layer) * E, h->h_ex.data() + size_t(layer) * E,
                            sizeof(pi::ExpertDev) * E, cudaMemcpyHostToDevice, st), "expert table");
    PI_CUDA(cudaStreamSynchronize(st), "load_layer sync");
    h->loaded[layer] = 1;
    if (h->prefill) pi::prefill_invalidate(h->prefill, layer);
    if (!h->vrm_ok.empty()) h->vrm_ok[layer] = 0;
    return PI_OK;
}

pi_status pi_ffn_set_hot_neurons(pi_ffn_t h, int hot_per_strip)
{
    if (!h) return fail(PI_ERR_INVALID_ARG, "null handle");
    for (char c : h->loaded)
        if (c) return fail(PI_ERR_INVALID_ARG, "set the VRAM budget before loading any layer");
    const int min_strip = h->desc.d_ff / h->S;
    if (hot_per_strip < 0 || hot_per_strip > min_strip)
        return fail(PI_ERR_INVALID_ARG, "hot_per_strip must be in [0, %d] (the smallest strip)", min_strip);
    h->hot_k = hot_per_strip;
    return PI_OK;
}

pi_status pi_neuron_table(pi_ffn_t h, int layer, int expert, int32_t *perm_host)
{
    if (!h || !perm_host) return fail(PI_ERR_INVALID_ARG, "pi_neuron_table: null argument");
    if (layer < 0 || layer >= h->desc.n_layers || expert < 0 || expert >= h->desc.n_experts)
        return fail(PI_ERR_INVALID_ARG, "layer/expert out of range");
    if (!h->loaded[layer]) return fail(PI_ERR_NOT_LOADED, "layer %d not loaded", layer);
    const auto &v = h->perm[size_t(layer) * h->desc.n_experts + expert];
    std::memcpy(perm_host, v.data(), sizeof(int32_t) * v.size());
    return PI_OK;
}

static pi::DecodeParams base_params(pi_ffn_t h)
{
    pi::DecodeParams p{};
    const pi_ffn_desc &D = h->desc;
    p.ex = h->d_ex;
    p.router = h->d_router;
    p.strip_off = h->d_strip_off;
    p.grp_off = h->d_grp_off;
    p.d = D.d_model;
    p.F = D.d_ff;
    p.r = D.rank;
    p.E = D.n_experts;
    p.top_k = D.top_k;
    p.act = int(D.act);
    p.gated = h->gated;
    p.S = h->S;
    p.threshold = D.threshold;
    p.eps = D.eps;
    p.vrow = h->vrow;
    p.urow = h->urow;
    p.wrow = h->wrow;
    p.gu_bytes = (h->gated ? 2 : 1) * h->wrow;
    p.spec_down = h->spec;
    p.rec_bytes = p.gu_bytes + (h->spec ? h->wrow : 0);
    p.wd_stride = h->spec ? p.rec_bytes : h->wrow;
    p.u_swz = h->u_swz;
    p.yfix = h->yfix;
    p.rbuf = h->rbuf;
    p.lists = h->lists;
    p.counts = h->counts;
    p.pub = h->pub;
    p.bar = h->bar;
    p.err = h->err;
    p.wait_ns = h->wait_ns;
    p.debug_flags = h->debug_flags;
    p.local_gather = (h->debug_flags & 4) ? 1 : 0;
    p.hot_k = h->hot_k;
    p.prof = h->prof;
    return p;
}

pi_status pi_predict(pi_ffn_t h, int layer, int expert, const float *x_dev, int32_t *idx_dev,
                     int32_t *count_dev, float *z_dev, void *stream)
{
    if (!h || !x_dev || !idx_dev || !count_dev) return fail(PI_ERR_INVALID_ARG, "pi_predict: null argument");
    const pi_ffn_desc &D = h->desc;
    if (layer < 0 || layer >= D.n_layers || expert < 0 || expert >= D.n_experts)
        return fail(PI_ERR_INVALID_ARG, "layer/expert out of range");
    if (!h->loaded[layer]) return fail(PI_ERR_NOT_LOADED, "layer %d not loaded", layer);
    if (!aligned16(x_dev)) return fail(PI_ERR_INVALID_ARG, "x_dev must be 16-byte aligned");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    PI_CUDA(cudaSetDevice(D.device), "cudaSetDevice");
    pi::DecodeParams p = base_params(h);
    p.mode = pi::kModePredict;
    p.pred_expert = expert;
    p.layer_begin = layer;
    p.layer_end = layer + 1;
    p.x_in = x_dev;
    p.z_out = z_dev;
    p.idx_out = idx_dev;
    p.count_out = count_dev;
    PI_CUDA(cudaMemsetAsync(h->bar, 0, sizeof(unsigned) * pi::kBarWords, st), "memset barrier");
    PI_CUDA(pi::launch_decode(h->wfmt, h->pfmt, p, st), "launch predict");
    return PI_OK;
}

pi_status pi_sparse_ffn_decode(pi_ffn_t h, int layer_begin, int layer_end, float *resid_dev,
                               float *trace_dev, int32_t *stats_dev, uint32_t *mask_dev, void *stream)
{
    if (!h || !resid_dev) return fail(PI_ERR_INVALID_ARG, "pi_sparse_ffn_decode: null argument");
    const pi_ffn_desc &D = h->desc;
    if (layer_begin < 0 || layer_end > D.n_layers || layer_begin >= layer_end)
        return fail(PI_ERR_INVALID_ARG, "layer range [%d, %d) invalid for %d layers", layer_begin,
                    layer_end, D.n_layers);
    for (int l = layer_begin; l < layer_end; ++l)
        if (!h->loaded[l]) return fail(PI_ERR_NOT_LOADED, "layer %d not loaded", l);
    if (!aligned16(resid_dev) || (trace_dev && !aligned16(trace_dev)))
        return fail(PI_ERR_INVALID_ARG, "resid_dev and trace_dev must be 16-byte aligned");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    PI_CUDA(cudaSetDevice(D.device), "cudaSetDevice");
    const int nl = layer_end - layer_begin;
    pi::DecodeParams p = base_params(h);
    p.mode = pi::kModeDecode;
    p.layer_begin = layer_begin;
    p.layer_end = layer_end;
    p.resid = resid_dev;
    p.trace = trace_dev;
    p.stats = stats_dev;
    p.masks = mask_dev;
    PI_CUDA(cudaMemsetAsync(h->bar, 0, sizeof(unsigned) * pi::kBarWords, st), "memset barrier");
    if (stats_dev) PI_CUDA(cudaMemsetAsync(stats_dev, 0, sizeof(int32_t) * 4 * nl, st), "memset stats");
    if (mask_dev)
        PI_CUDA(cudaMemsetAsync(mask_dev, 0, sizeof(uint32_t) * size_t(nl) * D.top_k * ((D.d_ff + 31) / 32), st),
                "memset masks");
    PI_CUDA(pi::launch_decode(h->wfmt, h->pfmt, p, st), "launch decode");
    return PI_OK;
}

pi_status pi_sparse_ffn_decode_batch(pi_ffn_t h, int layer_begin, int layer_end, int n_tokens,
                                     float *resid_dev, float *trace_dev, int32_t *stats_dev,
                                     uint32_t *mask_dev, void *stream)
{
    if (!h || !resid_dev) return fail(PI_ERR_INVALID_ARG, "pi_sparse_ffn_decode_batch: null argument");
    const pi_ffn_desc &D = h->desc;
    if (layer_begin < 0 || layer_end > D.n_layers || layer_begin >= layer_end)
        return fail(PI_ERR_INVALID_ARG, "layer range [%d, %d) invalid for %d layers", layer_begin,
                    layer_end, D.n_layers);
    if (n_tokens < 1 || n_tokens > 4 * pi::batch_max_tokens())
        return fail(PI_ERR_INVALID_ARG, "n_tokens must be in [1, %d]", 4 * pi::batch_max_tokens());
    for (int l = layer_begin; l < layer_end; ++l)
        if (!h->loaded[l]) return fail(PI_ERR_NOT_LOADED, "layer %d not loaded", l);
    if (!aligned16(resid_dev) || (trace_dev && !aligned16(trace_dev)))
        return fail(PI_ERR_INVALID_ARG, "resid_dev and trace_dev must be 16-byte aligned");
    if (D.n_experts != 1) return fail(PI_ERR_UNSUPPORTED, "small-batch decode takes dense FFN layers");
    if (h->hot_k) return fail(PI_ERR_UNSUPPORTED, "small-batch decode needs every record in HBM (no VRAM budget)");
    if (!((D.w_dtype == PI_F16 && D.pred_dtype == PI_F16) || (D.w_dtype == PI_BF16 && D.pred_dtype == PI_BF16)))
        return fail(PI_ERR_UNSUPPORTED, "small-batch decode takes F16 or BF16 weights with a predictor of the same format");
    if (D.d_model > pi::batch_max_d())
        return fail(PI_ERR_UNSUPPORTED, "small-batch decode takes d_model <= %d", pi::batch_max_d());
    if ((D.d_model / 8 + h->S - 1) / h->S * 8 > 256)
        return fail(PI_ERR_UNSUPPORTED, "small-batch decode needs d_model / n_strips <= 256 columns");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    PI_CUDA(cudaSetDevice(D.device), "cudaSetDevice");
    if (h->batch_fits < 0) {   // co-residency of the batch kernel, checked once per handle
        int nsm = 0;
        PI_CUDA(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, D.device), "cudaDeviceGetAttribute");
        const int per_sm = pi::batch_max_blocks_per_sm(h->wfmt);
        h->batch_fits = per_sm >= 1 && h->S <= per_sm * nsm ? 1 : 0;
    }
    if (!h->batch_fits)
        return fail(PI_ERR_UNSUPPORTED, "small-batch kernel: %d strips exceed co-resident CTAs", h->S);
    const int L = D.n_layers, S = h->S, d = D.d_model, r = D.rank, nbmax = pi::batch_max_tokens();
    const int tpl = pi::batch_tokens_per_launch(h->wfmt);
    // workspace: t [8 r] | ss [S 8] | partials [S 8 d] | counts [S] | pub [S kMaxStrip] | bar
    const size_t o_t = 0;
    const size_t o_ss = up256(o_t + sizeof(float) * size_t(nbmax) * r);
    const size_t o_part = up256(o_ss + sizeof(float) * size_t(S) * 8);
    const size_t o_cnt = up256(o_part + sizeof(float) * size_t(S) * nbmax * d);
    const size_t o_pub = up256(o_cnt + sizeof(int32_t) * S);
    const size_t o_bar = up256(o_pub + sizeof(unsigned long long) * size_t(S) * pi::kMaxStrip);
    const size_t total = up256(o_bar + sizeof(unsigned) * pi::kBarWords);
    if (!h->bscratch) {
        PI_CUDA(cudaMalloc(&h->bscratch, total), "cudaMalloc(batch workspace)");
        PI_CUDA(cudaMemset(h->bscratch, 0, total), "memset(batch workspace)");
        h->vrm_ok.assign(L, 0);
        PI_CUDA(cudaMalloc(&h->d_vrm, sizeof(uint8_t *) * L), "cudaMalloc(V table)");
        PI_CUDA(cudaMemset(h->d_vrm, 0, sizeof(uint8_t *) * L), "memset(V table)");
    }
    // the V table: each layer's V (row-major) for the range
    for (int l = layer_begin; l < layer_end; ++l) {
        if (h->vrm_ok[l]) continue;
        const uint8_t *vp = h->h_ex[size_t(l) * D.n_experts].V;
        PI_CUDA(cudaMemcpyAsync(h->d_vrm + l, &vp, sizeof(vp), cudaMemcpyHostToDevice, st), "V table");
        PI_CUDA(cudaStreamSynchronize(st), "V table sync");
        h->vrm_ok[l] = 1;
    }
    const int nl = layer_end - layer_begin;
    pi::BatchLaunch B{};
    B.ex = h->d_ex;
    B.vrm = h->d_vrm;
    B.strip_off = h->d_strip_off;
    B.grp_off = h->d_grp_off;
    B.d = d; B.F = D.d_ff; B.r = r; B.act = int(D.act); B.gated = h->gated; B.S = S; B.nb = n_tokens;
    B.layer_begin = layer_begin; B.layer_end = layer_end;
    B.threshold = D.threshold; B.eps = D.eps;
    B.vrow = h->vrow; B.urow = h->urow; B.wrow = h->wrow;
    B.gu_bytes = (h->gated ? 2 : 1) * h->wrow;
    B.spec = h->spec;
    B.rec_bytes = B.gu_bytes + (h->spec ? h->wrow : 0);
    B.wd_stride = h->spec ? B.rec_bytes : h->wrow;
    B.u_swz = h->u_swz;
    B.trace = trace_dev; B.stats = stats_dev; B.masks = mask_dev;
    B.ntok = n_tokens;
    B.t_buf = reinterpret_cast<float *>(h->bscratch + o_t);
    B.ss = reinterpret_cast<float *>(h->bscratch + o_ss);
    B.partials = reinterpret_cast<float *>(h->bscratch + o_part);
    B.counts = reinterpret_cast<int32_t *>(h->bscratch + o_cnt);
    B.pub = reinterpret_cast<unsigned long long *>(h->bscratch + o_pub);
    B.bar = reinterpret_cast<unsigned *>(h->bscratch + o_bar);
    B.err = h->err;
    B.wait_ns = h->wait_ns;
    if (stats_dev) PI_CUDA(cudaMemsetAsync(stats_dev, 0, sizeof(int32_t) * 4 * nl, st), "memset stats");
    if (mask_dev)
        PI_CUDA(cudaMemsetAsync(mask_dev, 0, sizeof(uint32_t) * size_t(nl) * n_tokens * ((D.d_ff + 31) / 32), st),
                "memset masks");
    // groups of up to eight (F16) or four (BF16) tokens, one launch each
    for (int t0 = 0; t0 < n_tokens; t0 += tpl) {
        B.tok0 = t0;
        B.nb = std::min(tpl, n_tokens - t0);
        B.resid = resid_dev + size_t(t0) * d;
        PI_CUDA(cudaMemsetAsync(B.bar, 0, sizeof(unsigned) * pi::kBarWords, st), "memset barrier");
        PI_CUDA(pi::launch_batch(h->wfmt, B, st), "launch batch decode");
    }
    return PI_OK;
}

namespace {
__global__ void k_residual_add(float *__restrict__ r, const float *__restrict__ y, int d)
{
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j < d) r[j] += y[j];
}
}  // namespace

pi_status pi_sparse_ffn_decode_partial(pi_ffn_t h, int layer, const float *resid_dev, float *y_dev,
                                       int32_t *stats_dev, uint32_t *mask_dev, void *stream)
{
    if (!h || !resid_dev || !y_dev) return fail(PI_ERR_INVALID_ARG, "pi_sparse_ffn_decode_partial: null argument");
    const pi_ffn_desc &D = h->desc;
    if (layer < 0 || layer >= D.n_layers) return fail(PI_ERR_INVALID_ARG, "layer %d out of range", layer);
    if (!h->loaded[layer]) return fail(PI_ERR_NOT_LOADED, "layer %d not loaded", layer);
    if (!aligned16(resid_dev) || !aligned16(y_dev))
        return fail(PI_ERR_INVALID_ARG, "resid_dev and y_dev must be 16-byte aligned");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    PI_CUDA(cudaSetDevice(D.device), "cudaSetDevice");
    pi::DecodeParams p = base_params(h);
    p.mode = pi::kModeDecode;
    p.layer_begin = layer;
    p.layer_end = layer + 1;
    p.resid = const_cast<float *>(resid_dev);   // read only: y goes to y_out
    p.y_out = y_dev;
    p.stats = stats_dev;
    p.masks = mask_dev;
    PI_CUDA(cudaMemsetAsync(h->bar, 0, sizeof(unsigned) * pi::kBarWords, st), "memset barrier");
    if (stats_dev) PI_CUDA(cudaMemsetAsync(stats_dev, 0, sizeof(int32_t) * 4, st), "memset stats");
    if (mask_dev)
        PI_CUDA(cudaMemsetAsync(mask_dev, 0, sizeof(uint32_t) * D.top_k * ((D.d_ff + 31) / 32), st), "memset masks");
    PI_CUDA(pi::launch_decode(h->wfmt, h->pfmt, p, st), "launch partial decode");
    return PI_OK;
}

pi_status pi_residual_add(pi_ffn_t h, float *resid_dev, const float *y_dev, void *stream)
{
    if (!h || !resid_dev || !y_dev) return fail(PI_ERR_INVALID_ARG, "pi_residual_add: null argument");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    PI_CUDA(cudaSetDevice(h->desc.device), "cudaSetDevice");
    const int d = h->desc.d_model;
    k_residual_add<<<(d + 255) / 256, 256, 0, st>>>(resid_dev, y_dev, d);
    PI_CUDA(cudaGetLastError(), "launch residual add");
    return PI_OK;
}

pi_status pi_sparse_ffn_decode_host(pi_ffn_t h, int layer_begin, int layer_end,
                                    const float *resid_in_host, float *resid_out_host, void *stream)
{
    if (!h || !resid_in_host || !resid_out_host)
        return fail(PI_ERR_INVALID_ARG, "pi_sparse_ffn_decode_host: null argument");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t bytes = sizeof(float) * h->desc.d_model;
    PI_CUDA(cudaSetDevice(h->desc.device), "cudaSetDevice");
    PI_CUDA(cudaMemcpyAsync(h->io, resid_in_host, bytes, cudaMemcpyHostToDevice, st), "copy in");
    pi_status s = pi_sparse_ffn_decode(h, layer_begin, layer_end, h->io, nullptr, nullptr, nullptr, stream);
    if (s != PI_OK) return s;
    PI_CUDA(cudaMemcpyAsync(resid_out_host, h->io, bytes, cudaMemcpyDeviceToHost, st), "copy out");
    PI_CUDA(cudaStreamSynchronize(st), "sync");
    return PI_OK;
}

pi_status pi_sync(pi_ffn_t h, void *stream)
{
    if (!h) return fail(PI_ERR_INVALID_ARG, "null handle");
    PI_CUDA(cudaSetDevice(h->desc.device), "cudaSetDevice");
    PI_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)), "stream sync");
    int err = 0;
    PI_CUDA(cudaMemcpy(&err, h->err, sizeof(int), cudaMemcpyDeviceToHost), "read error word");
    if (err == pi::kDevOk) return PI_OK;
    PI_CUDA(cudaMemset(h->err, 0, sizeof(int)), "clear error word");
    if (err == pi::kDevTimeout) return fail(PI_ERR_TIMEOUT, "a bounded device-side wait ran out");
    return fail(PI_ERR_DEVICE_CHECK, "device-side check failed (code %d)", err);
}

pi_status pi_debug_set(pi_ffn_t h, int flags, double wait_limit_s)
{
    if (!h) return fail(PI_ERR_INVALID_ARG, "null handle");
    if (!(wait_limit_s > 0.0) || wait_limit_s > 60.0)
        return fail(PI_ERR_INVALID_ARG, "wait_limit_s must be in (0, 60]");
    h->debug_flags = flags;
    h->wait_ns = static_cast<long long>(wait_limit_s * 1e9);
    return PI_OK;
}

pi_status pi_debug_phase_times(pi_ffn_t h, long long *times_dev)
{
    if (!h) return fail(PI_ERR_INVALID_ARG, "null handle");
    if (times_dev && (reinterpret_cast<uintptr_t>(times_dev) & 7u))
        return fail(PI_ERR_INVALID_ARG, "times_dev must be 8-byte aligned");
    h->prof = times_dev;
    return PI_OK;
}

pi_status pi_dense_ffn_prefill(pi_ffn_t h, int layer_begin, int layer_end, int n_tokens,
                               float *resid_dev, void *stream)
{
    if (!h || !resid_dev) return fail(PI_ERR_INVALID_ARG, "pi_dense_ffn_prefill: null argument");
    const pi_ffn_desc &D = h->desc;
    if (layer_begin < 0 || layer_end > D.n_layers || layer_begin >= layer_end)
        return fail(PI_ERR_INVALID_ARG, "layer range invalid");
    if (n_tokens < 1) return fail(PI_ERR_INVALID_ARG, "n_tokens must be >= 1");
    for (int l = layer_begin; l < layer_end; ++l)
        if (!h->loaded[l]) return fail(PI_ERR_NOT_LOADED, "layer %d not loaded", l);
    if (!aligned16(resid_dev)) return fail(PI_ERR_INVALID_ARG, "resid_dev must be 16-byte aligned");
    if (h->hot_k) return fail(PI_ERR_UNSUPPORTED, "dense prefill needs every record in HBM (no VRAM budget)");
    PI_CUDA(cudaSetDevice(D.device), "cudaSetDevice");
    pi::PrefillView v{};
    v.n_layers = D.n_layers;
    v.d = D.d_model;
    v.F = D.d_ff;
    v.E = D.n_experts;
    v.top_k = D.top_k;
    v.act = int(D.act);
    v.gated = h->gated;
    v.wfmt = h->wfmt;
    v.wrow = h->wrow;
    v.rec_bytes = (h->gated ? 2 : 1) * h->wrow + (h->spec ? h->wrow : 0);
    v.wd_stride = h->spec ? v.rec_bytes : h->wrow;
    v.eps = D.eps;
    v.ex = h->h_ex.data();
    v.router = h->router_mem.data();
    v.perm = &h->perm;
    v.err = h->err;
    v.wait_ns = h->wait_ns;
    v.debug_flags = h->debug_flags;
    char msg[256] = "";
    const int rc = pi::prefill_run(&h->prefill, v, layer_begin, layer_end, n_tokens, resid_dev,
                                   static_cast<cudaStream_t>(stream), msg, sizeof msg);
    if (rc == 1) return fail(PI_ERR_UNSUPPORTED, "%s", msg);
    if (rc == 2) return fail(PI_ERR_CUDA, "%s", msg);
    if (rc == 3) return fail(PI_ERR_OOM, "%s", msg);
    return PI_OK;
}

}  // extern "C"
