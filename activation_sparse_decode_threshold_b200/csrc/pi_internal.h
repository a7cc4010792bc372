// pi_internal.h -- structures shared by the host side of the C ABI and the
// sm_100a kernels.  Not part of the public interface.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace pi {

// Decode kernel geometry: one CTA of 16 warps per neuron strip, one strip per
// SM; every warp computes (weights reach the SM through L2 prefetches and
// batched 128-bit loads).
constexpr int kConsumerWarps = 16;
constexpr int kThreads = kConsumerWarps * 32;
constexpr int kMaxStrip = 256;        // neurons per strip (per CTA) at most
constexpr int kMaxStrips = 256;       // strips (CTAs) at most
constexpr int kMaxTopK = 2;
constexpr int kMaxExperts = 16;
constexpr int kMaxRankTotal = 2048;   // top_k * rank
constexpr int kStageBytes = 200 * 1024;   // shared-memory staging of V rows / U strips / gathered rows
constexpr int kMaxSliceCols = 1024;       // residual columns per CTA at most

enum Fmt { kF32 = 0, kF16 = 1, kBF16 = 2, kI4 = 3, kI8 = 4 };   // kI8: predictor only

// One expert (or dense FFN) of one layer, in table order, library-owned.
// A neuron's input record holds its W_gate row followed by its W_up row when
// gated (2 * wrow bytes), or its W_1 row when non-gated (wrow bytes), so one
// bulk copy brings everything the neuron's activation needs.  An INT4 row is
// its d/2 nibble bytes followed by its d/32 fp16 scales.
struct ExpertDev {
    const uint8_t *V;    // r rows of vrow bytes, row-major (rank is not permuted); each
                         // CTA reads its own run of rows for the t phase
    const uint8_t *U;    // F rows of urow bytes, table order
    const float *c;      // F biases, table order
    const uint8_t *Wgu;  // F neuron records, table order, rec_bytes apart: gate row (+ up row)
                         // (+ the W_down row for the speculative kinds)
    const uint8_t *Wd;   // F rows of wrow bytes, wd_stride apart: W_down columns, neuron-major
                         // (inside the records for the speculative kinds)
    const float *sU;     // 8-bit predictor: scale of each U row (table order); else null
    const float *sV;     // 8-bit predictor: scale of each V row (r); else null
    // With a VRAM budget (DecodeParams::hot_k > 0) Wgu / Wd hold only the first
    // hot_k records of each strip (index b * hot_k + loc) and the others sit in
    // pinned host memory at these device-visible addresses (index pos - (b+1) hot_k).
    const uint8_t *Wgu_cold;
    const uint8_t *Wd_cold;
};

enum Mode { kModeDecode = 0, kModePredict = 1 };

struct DecodeParams {
    const ExpertDev *ex;            // [n_layers * E]
    const uint8_t *const *router;   // [n_layers] E x d fp16, or null entries
    const int32_t *strip_off;       // [S + 1]
    const int32_t *grp_off;         // [S + 1] column slices, in 8-column groups (the columns
                                    // of r, y and the trace each CTA writes)
    int d, F, r, E, top_k, act, gated, S;
    int layer_begin, layer_end;
    float threshold, eps;
    int vrow, urow, wrow;           // row bytes: V (pred fmt), U (pred fmt), W (weight fmt)
    int gu_bytes;                   // bytes of a neuron's input record (2 * wrow gated)
    int spec_down;                  // prefetch down rows of all predicted-active neurons
    int rec_bytes;                  // bytes between neuron records (gate|up, plus the down row when spec_down)
    int wd_stride;                  // bytes between W_down rows (rec_bytes when spec_down, else wrow)
    int u_swz;                      // U rows stored chunk-permuted (repack_u_swizzled)
    int mode, pred_expert;
    // inputs / outputs
    float *resid;                   // [d] decode: in/out residual
    float *y_out;                   // [d] or null: one-layer call that emits y (the residual unchanged)
    const float *x_in;              // [d] predict: layer input
    float *trace;                   // [(l1-l0) * d] or null
    int32_t *stats;                 // [(l1-l0) * 4] or null (zeroed by the host)
    uint32_t *masks;                // [(l1-l0) * top_k * ceil(F/32)] or null (zeroed)
    float *z_out;                   // predict: [F] or null
    int32_t *idx_out, *count_out;   // predict
    // scratch (library-owned or caller-provided, see pi_host.cu)
    unsigned long long *yfix;       // [2 * d] decode: each layer's y summed in 64-bit fixed point
                                    // (2^-32 units), by layer parity; the kernel clears them itself
    float *rbuf;                    // [2 * d] decode: each layer's input r, by layer parity
    int32_t *lists;                 // [S * kMaxStrip]  (predict)
    int32_t *counts;                // [S] active count of each strip
    unsigned long long *pub;        // [S * kMaxTopK * kMaxStrip] published active entries (decode):
                                    // low word (slot << 24) | table position, high word the bias bits
    unsigned *bar;                  // [2] grid barrier: arrivals, generation; zeroed before launch
    int *err;                       // device error word (0 = ok)
    long long wait_ns;              // bound on every device-side wait
    int debug_flags;
    int local_gather;               // each CTA gathers its own strip's active neurons (no balance step)
    int hot_k;                      // records in HBM per strip (0 = all; others in host memory)
    long long *prof;                // [(l1-l0) * kProfPoints * S] phase timestamps, or null
};

// Phase timestamps recorded per layer and CTA when DecodeParams::prof is set.
// layer kinds (bits of the decode kernel's MODE parameter)
constexpr int kModeMoE = 1, kModeGated = 2, kModeSpec = 4, kModePred = 8;
// Synchronisation area, zeroed before every launch (kBarWords 32-bit words):
// word 0 is the grid barrier's arrival counter; words kRouterWord on hold the
// routed layers' router-logit totals (2 x kMaxExperts 64-bit fixed-point
// values, by layer parity); words kTagTWord on hold the rows of t as tagged
// 64-bit slots (the value's bits in the low half, the writing layer's tag in
// the high half).
constexpr int kRouterWord = 256;
constexpr int kTagTWord = 512;
constexpr int kBarWords = kTagTWord + 2 * kMaxRankTotal;
static_assert(kRouterWord + 4 * kMaxExperts <= kTagTWord, "router totals inside the zeroed barrier area");
constexpr int kProfPoints = 32;   // timestamps and cycle counters per layer and CTA

cudaError_t launch_decode(int wfmt, int pfmt, const DecodeParams &p, cudaStream_t stream);
int decode_max_blocks_per_sm(int wfmt, int pfmt, int d);

// Small-batch decode (pi_batch.cu): up to batch_max_tokens() tokens per launch.
struct BatchLaunch {
    const ExpertDev *ex;                 // [n_layers]
    const uint8_t *const *vrm;           // [n_layers] V row-major
    const int32_t *strip_off, *grp_off;  // [S + 1]
    int d, F, r, act, gated, S, nb;
    int layer_begin, layer_end;
    float threshold, eps;
    int vrow, urow, wrow, gu_bytes, rec_bytes, wd_stride, spec, u_swz;
    float *resid, *trace;                // resid: this launch's nb rows; trace: all ntok rows per layer
    int32_t *stats;
    uint32_t *masks;                     // all ntok rows per layer
    int ntok, tok0;                      // tokens of the call, first token of this launch
    float *t_buf, *ss, *partials;        // [nb x r], [S x 8], [S x nb x d]
    int32_t *counts;                     // [S]
    unsigned long long *pub;             // [S x kMaxStrip]
    unsigned *bar;                       // [kBarWords], zeroed before launch
    int *err;
    long long wait_ns;
};
cudaError_t launch_batch(int wfmt, const BatchLaunch &L, cudaStream_t st);
int batch_max_blocks_per_sm(int wfmt);
int batch_max_tokens();
int batch_tokens_per_launch(int wfmt);   // 8 (F16), 4 (BF16: x and h as two bf16 parts)
int batch_max_d();
// Load-time repack kernels (pi_repack.cu).  repack_rows: dst record p is the
// concatenation of row perm[p] of each of the n_src sources (row bytes each a
// multiple of 16).
constexpr int kMaxRepackSrc = 6;
// dst_stride: bytes between records (0 = the records' own size).
cudaError_t repack_rows(uint8_t *dst, const int32_t *perm, int rows, int n_src,
                        const uint8_t *const *src, const int *row_bytes, cudaStream_t s,
                        long long dst_stride = 0);
cudaError_t repack_bias(const float *src, float *dst, const int32_t *perm, int n, cudaStream_t s);
// Records (`bytes` each, table order) split by strip position: the first hot_k
// of each strip to `hot`, the others to `cold` (a device-visible host buffer).
cudaError_t split_records(const uint8_t *src, uint8_t *hot, uint8_t *cold, int F, int bytes,
                          const int32_t *strip_off, int S, int hot_k, cudaStream_t s);
// U rows in table order, 16-byte chunks permuted inside each 128-byte group by
// (row - strip start) mod 8 (row_bytes a multiple of 128); strip_off on the device.
cudaError_t repack_u_swizzled(uint8_t *dst, const int32_t *perm, int rows, const uint8_t *src, int row_bytes,
                              const int32_t *strip_off, int S, cudaStream_t s);
// dst_stride_bytes: bytes between neuron rows (0 = d * elem_bytes).
cudaError_t repack_down_transpose(const uint8_t *w_down, uint8_t *dst, const int32_t *perm,
                                  int d, int F, int elem_bytes, cudaStream_t s, long long dst_stride_bytes = 0);

// Sets the message returned by pi_last_error on this host thread.
void set_last_error(const char *msg);

// Device error codes written into the error word.
enum DevErr { kDevOk = 0, kDevTimeout = 1, kDevCheck = 2 };

}  // namespace pi
