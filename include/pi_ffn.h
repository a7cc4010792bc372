/*
 * pi_ffn.h -- C ABI of the predictor-guided, neuron-aware sparse FFN library
 * for NVIDIA B200 (sm_100a).
 *
 * What it computes (per decode token, per FFN layer), after the pages on
 * PowerInfer and PowerInfer-2:
 *   x = RMSNorm(r)                                   (no weight, eps)
 *   [MoE] two experts from a softmax router           (TurboSparse-Mixtral-shaped layer)
 *   t = V x ; z = U t - c ; neuron i active iff z_i > threshold
 *        -- the online activation predictor: "PowerInfer: fast LLM serving
 *           with a consumer-grade GPU" (unite.ai), sections "Online phase" and
 *           "Adaptive sparse predictor"; nearauto.com PowerInfer article,
 *           "PowerInfer architecture", Fig. 8.
 *   for active i only: g = W_gate[i].x - c_i, u = W_up[i].x, h = act(g, u)
 *   y = sum over active i with h_i != 0 of h_i * W_down[:, i]
 *        -- neuron-aware operators over rows of the input matrices and
 *           columns of the output matrix, no dense conversion: unite.ai,
 *           "Neuron-aware operators".
 *   r <- r + y
 * Neurons are stored in neuron-table order ("Neuron placement and
 * management", unite.ai): the table maps each stored position to the
 * neuron's original index, and results are returned in original d_model order.
 *
 * Conventions for every call:
 *  - Pointers marked _dev are CUDA device pointers owned by the caller; _host
 *    are host pointers.  Nothing here takes or returns a torch type.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Device work is enqueued on it and the call returns without waiting,
 *    unless the call says otherwise.
 *  - Arguments are validated before any work is enqueued; on a bad argument
 *    the call returns PI_ERR_INVALID_ARG (or PI_ERR_UNSUPPORTED) and enqueues
 *    nothing.  pi_last_error() then describes the problem.
 *  - Faults found on the device (a bounded wait that ran out, a bad index)
 *    never trap: the kernel records an error word and returns; pi_sync()
 *    reports it.  No call aborts, throws or exits the process.
 *  - One handle may be used from one host thread at a time.  Calls that
 *    overlap on the GPU (two streams, same handle) race on the handle's
 *    scratch memory and must not be issued.
 */
#ifndef PI_FFN_H
#define PI_FFN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PI_API __attribute__((visibility("default")))
#else
#define PI_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pi_ffn *pi_ffn_t;

typedef enum {
    PI_OK = 0,
    PI_ERR_INVALID_ARG = 1,   /* bad pointer, size, index or combination */
    PI_ERR_UNSUPPORTED = 2,   /* valid but not implemented for this shape/format */
    PI_ERR_OOM = 3,           /* device allocation failed */
    PI_ERR_CUDA = 4,          /* a CUDA runtime call failed */
    PI_ERR_TIMEOUT = 5,       /* a bounded device-side wait ran out */
    PI_ERR_DEVICE_CHECK = 6,  /* a device-side consistency check failed */
    PI_ERR_NOT_LOADED = 7     /* a layer in the range was never loaded */
} pi_status;

/* Activation of the FFN (h as a function of g = W_gate.x - c and u = W_up.x).
 * RELU is non-gated: the layer has one input matrix, passed as w_gate
 * (W_1), and h = max(g, 0).  REGLU: h = max(g, 0) * u.  DRELU: h = max(g, 0)
 * * max(u, 0) (citnews.com.cn PowerInfer-2 article, dReLU replaces SwiGLU). */
typedef enum { PI_ACT_RELU = 0, PI_ACT_REGLU = 1, PI_ACT_DRELU = 2 } pi_act;

/* Stored formats.  INT4G32: symmetric 4-bit, value = s * (n - 8) with n the
 * nibble (low nibble = even element) and s one fp16 scale per 32 consecutive
 * elements of a neuron vector (a W_gate/W_up row or a W_down column).
 * I8 (predictor only): symmetric 8-bit, value = s * q with q a signed byte and
 * s one fp32 scale per row of U and of V -- the cheaper predictor (predictors
 * are costly in memory: PowerInfer (unite.ai), "Adaptive sparse predictor"),
 * half the bytes of a 16-bit one. */
typedef enum { PI_F32 = 0, PI_F16 = 1, PI_BF16 = 2, PI_INT4G32 = 3, PI_I8 = 4 } pi_dtype;

typedef struct {
    int n_layers;        /* layers in the stack, >= 1 */
    int d_model;         /* d: multiple of 256, <= 8192 (<= 4096 for F32) */
    int d_ff;            /* F: neurons per FFN (per expert), <= 256 * n_strips */
    int rank;            /* predictor rank r: a multiple of 16 (the tensor-core
                            predictor dots take 16 columns per step; 32 for
                            an I8 predictor, whose integer dots take 32),
                            r <= 1024 (<= 512 for F32) */
    int n_experts;       /* 1 = dense FFN; 2..16 = MoE with top-2 routing */
    int top_k;           /* 1 for a dense FFN, 2 for MoE */
    pi_act act;
    pi_dtype w_dtype;    /* F32, F16, BF16 or INT4G32 */
    pi_dtype pred_dtype; /* F32, F16, BF16 or I8 (F32 weights need F32 here; I8 goes
                            with F16, BF16 or INT4G32 weights) */
    int n_strips;        /* neuron strips per FFN = CTAs of the decode kernel;
                            0 = number of SMs of the device */
    float threshold;     /* predictor threshold, normally 0 (active iff z > threshold) */
    float eps;           /* RMSNorm epsilon, normally 1e-6 */
    int device;          /* CUDA device ordinal */
} pi_ffn_desc;

/* Weights of one FFN or one MoE expert, in ORIGINAL neuron order, as device
 * pointers (read during pi_ffn_load_layer only; the caller keeps ownership).
 *   w_gate  F x d row-major (W_1 when non-gated)        [w_dtype]
 *   w_up    F x d row-major, NULL when non-gated          [w_dtype]
 *   w_down  float formats: d x F row-major (nn.Linear layout);
 *           INT4G32: neuron-major F x d (row i = column i of W_down)
 *   s_gate, s_up, s_down  INT4G32 only: F x d/32 fp16 scales (one per 32
 *           consecutive elements of each neuron vector); NULL otherwise.
 *           INT4 matrices are F x d/2 bytes of nibbles.
 *   bias    c, F floats (the gate bias enters as -c)
 *   U       F x r row-major [pred_dtype];  V  r x d row-major [pred_dtype]
 *   s_U, s_V  I8 predictor only: fp32 scale of each row of U (F) and of V (r);
 *           NULL otherwise.
 */
typedef struct {
    const void *w_gate, *w_up, *w_down;
    const void *s_gate, *s_up, *s_down;
    const float *bias;
    const void *U, *V;
    const float *s_U, *s_V;
} pi_expert_weights;

/* Create a handle: validates `desc`, reserves per-handle scratch on
 * desc->device.  No weights yet.  Returns PI_OK and *out, or an error. */
PI_API pi_status pi_ffn_create(const pi_ffn_desc *desc, pi_ffn_t *out);

/* Load layer `layer` (0 <= layer < n_layers): builds each expert's neuron
 * table from `freq_host` (n_experts x F profiled firing frequencies, NULL =
 * identity table), then copies and repacks the weights into library-owned
 * device memory in table order (rows of W_gate, W_up, U and c permuted;
 * W_down transposed so each neuron's column is contiguous; INT4 scales stored
 * after each neuron's nibbles).  `experts` has n_experts entries.  `router_dev`
 * is the E x d fp16 router for MoE (NULL for a dense FFN).  Work runs on
 * `stream`; the call synchronises it before returning, so the caller's
 * buffers may be freed afterwards.  Reloading a layer replaces it. */
PI_API pi_status pi_ffn_load_layer(pi_ffn_t h, int layer, const pi_expert_weights *experts,
                            const void *router_dev, const float *freq_host, void *stream);

/* VRAM budget (the survey's "next" row f4; PowerInfer (unite.ai), "Neuron
 * placement and management": hot neurons on the GPU, cold ones in host memory).
 * Keep only the first `hot_per_strip` neuron records of every strip in device
 * memory -- the strip's hottest neurons, since the table orders each strip
 * hottest first -- and the others in pinned, device-mapped host memory, read
 * by the decode kernel over the host link when predicted active.  The
 * predictor (V, U, c) and INT4 scales stay in device memory.  0 (the default)
 * keeps every record in device memory.  Must be called before any layer is
 * loaded; 0 <= hot_per_strip <= floor(d_ff / n_strips), else
 * PI_ERR_INVALID_ARG.  Decode results are bit-identical to a handle without a
 * budget; pi_dense_ffn_prefill and pi_sparse_ffn_decode_batch return
 * PI_ERR_UNSUPPORTED on a budgeted handle.  Device memory per layer and expert
 * drops by (d_ff - n_strips * hot_per_strip) records. */
PI_API pi_status pi_ffn_set_hot_neurons(pi_ffn_t h, int hot_per_strip);

/* Neuron table of (layer, expert): perm_host[p] = original index of the
 * neuron stored at table position p (F entries).  Strip b of the table holds
 * positions [off[b], off[b+1]) with off from pi_strip_offsets.  Table rule:
 * neurons ranked by descending frequency (ties: lower index first), dealt to
 * the strips in snake order (round j ascending for even j, descending for odd
 * j; a full strip is skipped); a strip keeps its neurons hottest first. */
PI_API pi_status pi_neuron_table(pi_ffn_t h, int layer, int expert, int32_t *perm_host);

/* Strip offsets (n_strips + 1 entries): strip b holds floor(F/S) + (b < F mod S)
 * neurons.  n_strips is also returned through *n_strips_out when non-NULL. */
PI_API pi_status pi_strip_offsets(pi_ffn_t h, int32_t *off_host, int *n_strips_out);

/* Predictor alone for (layer, expert) on a given layer input x (already
 * normalised, d floats):
 *   idx_dev    [F] int32: the active neurons' TABLE positions, ascending
 *              (map back with pi_neuron_table); entries past *count unspecified
 *   count_dev  [1] int32: number of active neurons
 *   z_dev      [F] float or NULL: predictor logits z in table order
 * Uses the same device code as the predictor inside pi_sparse_ffn_decode. */
PI_API pi_status pi_predict(pi_ffn_t h, int layer, int expert, const float *x_dev,
                     int32_t *idx_dev, int32_t *count_dev, float *z_dev, void *stream);

/* Batch-1 sparse decode of layers [layer_begin, layer_end) on one token.
 *   resid_dev   [d] float, in/out: the residual stream r; on return r after
 *               the last layer.
 *   trace_dev   [(l1-l0) x d] float or NULL: the residual entering each layer.
 *   stats_dev   [(l1-l0) x 4] int32 or NULL: per layer {predicted-active
 *               neurons, neurons with h != 0, first expert, second expert}
 *               (counts summed over the used experts; experts -1 if dense).
 *   mask_dev    [(l1-l0) x top_k x ceil(F/32)] uint32 or NULL: predicted-active
 *               bits in table order (bit p%32 of word p/32), per used expert
 *               in ascending expert index.
 * All layers run in one persistent kernel with one CTA per strip.  The result
 * is deterministic: the same inputs give bit-identical outputs, and splitting
 * the range into several calls gives the same bits as one call. */
PI_API pi_status pi_sparse_ffn_decode(pi_ffn_t h, int layer_begin, int layer_end, float *resid_dev,
                               float *trace_dev, int32_t *stats_dev, uint32_t *mask_dev,
                               void *stream);

/* Small-batch sparse decode of layers [layer_begin, layer_end) on n_tokens
 * independent tokens (1 <= n_tokens <= 32), one persistent launch per group
 * of up to 8 tokens (F16 weights) or 4 tokens (BF16 weights).  The
 * sparse path keeps its gains at small batch sizes (nearauto.com PowerInfer
 * article, "Experiments", Fig. 14): per layer each token is normalised and
 * predicted on its own, the rows read are those of the UNION of the tokens'
 * predicted sets (each union neuron's W_gate / W_up / W_down rows fetched once
 * for the batch), and token b keeps its own predicted set (h exactly 0
 * outside it), so its output is its batch-1 output up to rounding.
 *   resid_dev  [n_tokens x d] float, in/out (row b = token b's residual).
 *   trace_dev  [(l1-l0) x n_tokens x d] float or NULL: each layer's input.
 *   stats_dev  [(l1-l0) x 4] int32 or NULL: per layer {union size, sum over the
 *              tokens of their predicted-active counts, union neurons with
 *              h != 0 for some token, 0}; with more tokens than one launch
 *              takes, the union figures are summed over the launches.
 *   mask_dev   [(l1-l0) x n_tokens x ceil(F/32)] uint32 or NULL: each token's
 *              predicted-active bits in table order.
 * Gate/up/down products run on the tensor cores with x and h rounded to fp16
 * for F16 weights (as in the dense prefill) and carried as two bf16 parts for
 * BF16 weights; the predictor keeps t and x to fp32 accuracy (16-bit parts).  Deterministic.  Supported: dense FFN layers
 * (n_experts = 1) with F16 or BF16 weights and a predictor of the same format,
 * d_model <= 4096 and d_model / n_strips <= 256; otherwise
 * PI_ERR_UNSUPPORTED.  The first call on a handle allocates a workspace
 * (about n_strips x 8 x d_model x 4 bytes) and a row-major copy of each used
 * layer's V (rank x d_model), kept until pi_ffn_destroy (a reloaded layer's
 * copy is remade).  Errors as pi_sparse_ffn_decode, plus PI_ERR_INVALID_ARG
 * for n_tokens outside [1, 32]. */
PI_API pi_status pi_sparse_ffn_decode_batch(pi_ffn_t h, int layer_begin, int layer_end, int n_tokens,
                                            float *resid_dev, float *trace_dev, int32_t *stats_dev,
                                            uint32_t *mask_dev, void *stream);

/* Tensor-parallel neuron sharding (the survey's "next" row f3; the pages name
 * no collective).  A handle may hold a SHARD of each layer's neurons: its
 * d_ff is the shard's neuron count and pi_ffn_load_layer receives that
 * shard's rows of W_gate / W_up / U / c and columns of W_down, with the full
 * V (replicated), so each shard predicts exactly its own neurons of the full
 * predictor.  The layer's output y is the sum over the shards.
 *
 * pi_sparse_ffn_decode_partial runs one layer on resid_dev (the residual
 * entering the layer, [d] float, read only) and writes this handle's share of
 * y to y_dev ([d] float): RMSNorm, prediction, gather and the fixed-point
 * merge of the CTAs' partials as in pi_sparse_ffn_decode, without the
 * residual add.  The caller
 * sums y over the shards (an all-reduce across ranks, e.g. NCCL) and adds it
 * with pi_residual_add (resid_dev[j] += y_dev[j], j < d).  A handle holding
 * all neurons gives exactly y of pi_sparse_ffn_decode's layer.  stats_dev
 * ([4]) and mask_dev (top_k x ceil(d_ff/32)) as in pi_sparse_ffn_decode, for
 * this shard.  Asynchronous on `stream`; errors as pi_sparse_ffn_decode. */
PI_API pi_status pi_sparse_ffn_decode_partial(pi_ffn_t h, int layer, const float *resid_dev, float *y_dev,
                                              int32_t *stats_dev, uint32_t *mask_dev, void *stream);
PI_API pi_status pi_residual_add(pi_ffn_t h, float *resid_dev, const float *y_dev, void *stream);

/* Same as pi_sparse_ffn_decode on HOST buffers: copies resid_in_host (d
 * floats) to the device, decodes, copies the result to resid_out_host, and
 * synchronises `stream` before returning.  Host buffers should be pinned for
 * the copies to run at full speed.  The two may alias. */
PI_API pi_status pi_sparse_ffn_decode_host(pi_ffn_t h, int layer_begin, int layer_end,
                                    const float *resid_in_host, float *resid_out_host,
                                    void *stream);

/* Dense multi-token prefill of layers [layer_begin, layer_end) on the tensor
 * cores (PowerInfer-2: prefill activates almost every neuron and runs as large
 * dense clusters; citnews.com.cn article, "Neuron-cluster heterogeneous
 * computing").  resid_dev is n_tokens x d float, in/out.  Per layer every
 * token is normalised, routed (MoE), and passed through the full FFN of its
 * expert(s) with no predictor; outputs are combined in ascending expert index
 * and added to the residual.  resid_dev is 16-byte aligned and caller-owned;
 * the library owns a workspace that grows to the largest n_tokens seen (about
 * n_tokens x (4 d_ff + 38 d_model) bytes).  Work is asynchronous on
 * `stream`; pi_sync reports device-side errors.  The result is deterministic
 * and each token's row depends only on that token.
 * Errors: PI_ERR_INVALID_ARG (null pointer, bad layer range, n_tokens < 1,
 * misaligned resid_dev), PI_ERR_NOT_LOADED (a layer of the range not loaded),
 * PI_ERR_UNSUPPORTED (weights other than F16/BF16/INT4G32, or d_ff not a
 * multiple of 128), PI_ERR_OOM (workspace), PI_ERR_CUDA. */
PI_API pi_status pi_dense_ffn_prefill(pi_ffn_t h, int layer_begin, int layer_end, int n_tokens,
                               float *resid_dev, void *stream);

/* Wait for `stream` and report (then clear) the handle's device error word:
 * PI_OK, PI_ERR_TIMEOUT or PI_ERR_DEVICE_CHECK. */
PI_API pi_status pi_sync(pi_ffn_t h, void *stream);

/* Message for the last non-OK status returned on this host thread. */
PI_API const char *pi_last_error(void);

/* Release the handle and all device memory it owns (after its work is done). */
PI_API void pi_ffn_destroy(pi_ffn_t h);

/* Testing aid: bound every device-side wait of this handle (decode and
 * prefill kernels) by `wait_limit_s` seconds (default 2.0).  With flags &
 * PI_DEBUG_STALL_BARRIER, the decode kernel's first grid barrier waits for one
 * arrival that never comes; with flags & PI_DEBUG_STALL_T_POLL, every CTA of
 * the decode kernel polls the rows of t of its first layer for a tag that no
 * CTA writes; with flags & PI_DEBUG_STALL_PREFILL, one producer thread of the
 * first prefill gate/up GEMM tile never publishes its first stage, so the
 * tensor-core issuer's bounded wait runs out before it issues any MMA.  Either
 * way the wait runs out, the kernel releases what it holds (in-flight copies,
 * tensor memory) and returns, and pi_sync reports PI_ERR_TIMEOUT; the handle
 * stays usable.  (Flag 4 is taken: each CTA gathers its own strip's active
 * neurons, without the balance step.) */
#define PI_DEBUG_STALL_BARRIER 1
#define PI_DEBUG_STALL_PREFILL 2
#define PI_DEBUG_STALL_T_POLL 8
PI_API pi_status pi_debug_set(pi_ffn_t h, int flags, double wait_limit_s);

/* Testing aid: when `times_dev` is non-NULL, each later pi_sparse_ffn_decode
 * call records, per layer and CTA, %globaltimer (ns) at these points k:
 *   0 layer start, 1 layer t polled and biases ready, 14 first predictor rows in
 *   shared memory, 15 first tensor-core logits done, 9 predictor logits done,
 *   2 active list done, 16 after the balance barrier, 8 this CTA's share of
 *   the active list known, 17 first gathered rows landed, 25 gather rounds
 *   done, 26 down rows done (the CTA's partial of y complete), 3 partial
 *   merged into the layer's total, 4 after the merge barrier, 20 next input
 *   summed, 7 next x formed, 5 this CTA's rows of t written, 6 the input
 *   step done (the prologue's grid barrier included); for routed (MoE)
 *   layers also 22 router share added, 23 after the router barrier, 18
 *   experts chosen, 19 first V rows in shared memory;
 * and k = 10..13 the clock cycles thread 0 spent obtaining the layer input,
 * waiting for predictor rows, waiting for gathered rows and waiting in grid
 * barriers.  Points 20, 7, 22, 23, 18, 19, 5 and 6 belong to the step that
 * forms the NEXT layer's input, recorded under the layer just run.  Value
 * (layer - layer_begin, k, cta) sits at
 * times_dev[((layer - layer_begin) * 32 + k) * n_strips + cta].  The buffer
 * (caller-owned, device, 8-byte aligned) must hold (l1 - l0) * 32 * n_strips
 * values.  NULL turns recording off. */
PI_API pi_status pi_debug_phase_times(pi_ffn_t h, long long *times_dev);

/* The low-rank predictor on caller-owned weights, with no device allocation
 * (no counterpart in the pages: it exists for callers that cannot call
 * cudaMalloc where they predict -- a serving loop whose device memory is fully
 * committed at start-up, a host runtime that owns the allocator, or code with
 * no pi_ffn handle, whose creation allocates).
 *   V_dev r x d, U_dev F x r (row-major, ORIGINAL neuron order, pred_dtype),
 *   bias_dev F floats, x_dev d floats (the layer input, already normalised);
 *   V, U and x 16-byte aligned.  Outputs as pi_predict, with table position =
 *   original index: idx_dev [F] active neurons ascending, count_dev [1],
 *   z_dev [F] logits or NULL.
 * Limits: d_model a multiple of 256, <= 8192 (<= 4096 for F32); rank as in
 * pi_ffn_desc; d_ff <= 256 * min(SM count, 256); larger sizes return
 * PI_ERR_INVALID_ARG.  Scratch: one file-scope __device__ array of about 300 KB
 * that every device loading the library holds until exit.
 * Runs on the current device, which must be one of devices 0..63 (a higher
 * index returns PI_ERR_UNSUPPORTED).  Its first call on a device looks up the
 * array's device address (cudaGetSymbolAddress) and must come before any
 * stream capture on that device; the address is kept for the life of the
 * process, so cudaDeviceReset must not be called on a device after this entry
 * point has been used there.  Every call shares the array and leaves its
 * contents behind (each call clears what must start at zero), so calls that
 * overlap on the GPU -- on two streams, or from two threads -- race and must
 * not be issued.  *count_dev reads -1 if any bounded wait of the call ran out
 * (a second, one-thread kernel on `stream` writes it after the predictor).
 * Asynchronous on `stream`. */
PI_API pi_status pi_predict_noalloc(int d_model, int d_ff, int rank, pi_dtype pred_dtype,
                                    float threshold, const void *V_dev, const void *U_dev,
                                    const float *bias_dev, const float *x_dev, int32_t *idx_dev,
                                    int32_t *count_dev, float *z_dev, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* PI_FFN_H */
