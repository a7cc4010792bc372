/*
 * oracle.c -- plain fp64 CPU restatement of the predictor-guided, neuron-aware
 * sparse FFN of batch-1 decode (PowerInfer / PowerInfer-2).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the correctness oracle: it is called
 * by the tests, by __graft_entry__.smoke() and by bench.py's CPU-baseline leg,
 * and by nothing else.  It shares no code, header, table or constant with the
 * CUDA library under activation_sparse_decode_threshold_b200/csrc, and the
 * library never calls it.  Every sum is a plain ascending loop in double
 * precision; OpenMP only splits loops whose iterations are independent
 * (one neuron's dot product, one output element's sum), so no sum is
 * reordered.
 *
 * Sources (page title, section):
 *  [PI-unite]  "PowerInfer: fast large language model serving with a consumer-
 *              grade GPU" (unite.ai) -- sections "Online phase: neuron-aware
 *              LLM inference engine", "Adaptive sparse predictor", "Neuron
 *              placement and management", "Neuron-aware operators".
 *  [PI-arch]   "Is the 4090 a replacement for the A100? ..." (nearauto.com) --
 *              section "PowerInfer architecture", Fig. 8.
 *  [PI2-news]  "PowerInfer-2 ... 47B model on a phone" (citnews.com.cn) --
 *              sections "Dynamic neuron cache", "Neuron-cluster heterogeneous
 *              computing", "Raising sparsity at low cost" (dReLU).
 *  [PI2-rev]   "PowerInfer-2: Fast Large Language Model Inference on a
 *              Smartphone" (nubint.ai review) -- "Proposed method".
 *
 * Readings where the pages are silent (each is also listed in the design
 * notes): the predictor is the low-rank pair z = U (V x) - c; a neuron is
 * active iff z > 0; the FFN bias -c sits on the gate (on W_1 when non-gated);
 * dReLU = relu(gate) * relu(up); RMSNorm has no weight and eps = 1e-6; INT4 is
 * symmetric group-32 (nibble n = q + 8, low nibble = even element, fp16 scale
 * per 32 consecutive elements of a neuron vector); MoE routing is softmax over
 * the experts, top-2 (ties to the lower index), weights renormalised over the
 * two.  The cheaper predictor format (I8ROW) is symmetric 8-bit with one fp32
 * scale per row: element k of row i is s_i * q_ik, q_ik a signed byte.
 *
 * Parity status: every function below is pinned by tests/test_oracle_pins.py
 * (closed forms, brute force on 8-neuron layers, the Fig. 8 merge, independent
 * numpy restatements of special cases, hand-packed INT4 and IEEE bit patterns).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { OR_F32 = 0, OR_F16 = 1, OR_BF16 = 2, OR_INT4G32 = 3, OR_I8ROW = 4 };
enum { OR_RELU = 0, OR_REGLU = 1, OR_DRELU = 2 };

/* ---------------------------------------------------------------------------
 * Number formats.
 * ------------------------------------------------------------------------- */

/* IEEE 754 binary16 -> double, from the format's definition:
 * sign(1) exponent(5, bias 15) fraction(10); exponent 0 = subnormal. */
double or_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 0x1f;
    int frac = h & 0x3ff;
    double v;
    if (expo == 0)
        v = ldexp((double)frac, -24);                 /* frac * 2^-10 * 2^-14 */
    else if (expo == 31)
        v = frac ? NAN : INFINITY;
    else
        v = ldexp(1.0 + (double)frac / 1024.0, expo - 15);
    return sign ? -v : v;
}

/* bfloat16 -> double: bfloat16 is the top 16 bits of an IEEE binary32. */
double or_bf16_to_double(uint16_t b)
{
    uint32_t bits = (uint32_t)b << 16;
    float f;
    memcpy(&f, &bits, 4);
    return (double)f;
}

/* One element of a stored float matrix (row-major, n columns). */
static double or_elem(int dtype, const void *base, long idx)
{
    switch (dtype) {
    case OR_F32:  return (double)((const float *)base)[idx];
    case OR_F16:  return or_half_to_double(((const uint16_t *)base)[idx]);
    case OR_BF16: return or_bf16_to_double(((const uint16_t *)base)[idx]);
    }
    return NAN;
}

/* INT4 group-32 dequantisation of one neuron vector of n elements:
 * element k has nibble n_k (low nibble of byte k/2 for even k, high nibble for
 * odd k) and value s_{k/32} * (n_k - 8).  Scales are fp16 bit patterns. */
void or_dequant_int4_g32(const uint8_t *q, const uint16_t *scales, int n,
                         double *out)
{
    for (int k = 0; k < n; ++k) {
        int byte = q[k / 2];
        int nib = (k % 2 == 0) ? (byte & 0xf) : (byte >> 4);
        out[k] = or_half_to_double(scales[k / 32]) * (double)(nib - 8);
    }
}

/* Row `row` of a stored matrix with n columns, as doubles.  For INT4 the
 * matrix is `rows x n/2` bytes of nibbles plus `rows x n/32` fp16 scales; for
 * I8ROW it is `rows x n` signed bytes plus one fp32 scale per row. */
void or_load_row(int dtype, const void *base, const void *scales, long row,
                 int n, double *out)
{
    if (dtype == OR_I8ROW) {
        const int8_t *q = (const int8_t *)base + row * (long)n;
        double s = (double)((const float *)scales)[row];
        for (int k = 0; k < n; ++k)
            out[k] = s * (double)q[k];
        return;
    }
    if (dtype == OR_INT4G32) {
        or_dequant_int4_g32((const uint8_t *)base + row * (long)(n / 2),
                            (const uint16_t *)scales + row * (long)(n / 32), n,
                            out);
        return;
    }
    for (int k = 0; k < n; ++k)
        out[k] = or_elem(dtype, base, row * (long)n + k);
}

/* ---------------------------------------------------------------------------
 * Layer input: parameterless RMSNorm, x = r / sqrt(mean(r^2) + eps).
 * ------------------------------------------------------------------------- */
void or_rmsnorm(const double *r, int d, double eps, double *x)
{
    double ss = 0.0;
    for (int j = 0; j < d; ++j)
        ss += r[j] * r[j];
    double inv = 1.0 / sqrt(ss / (double)d + eps);
    for (int j = 0; j < d; ++j)
        x[j] = r[j] * inv;
}

/* ---------------------------------------------------------------------------
 * Online activation predictor [PI-unite "Adaptive sparse predictor";
 * PI-arch Fig. 8]: identify the neurons of the layer likely to fire.
 * Low-rank form: t = V x (V is rank x d), z_i = U_i . t - c_i (U is F x rank),
 * neuron i predicted active iff z_i > threshold (threshold 0 by default).
 * ------------------------------------------------------------------------- */
void or_predict_q(int d, int F, int rank, int pdtype, const void *V,
                  const void *V_s, const void *U, const void *U_s,
                  const double *c, double threshold, const double *x,
                  double *t, double *z, uint8_t *mask)
{
    #pragma omp parallel for schedule(static)
    for (int k = 0; k < rank; ++k) {
        double *row = (double *)malloc(sizeof(double) * d);
        or_load_row(pdtype, V, V_s, k, d, row);
        double acc = 0.0;
        for (int j = 0; j < d; ++j)
            acc += row[j] * x[j];
        t[k] = acc;
        free(row);
    }
    #pragma omp parallel for schedule(static)
    for (int i = 0; i < F; ++i) {
        double *row = (double *)malloc(sizeof(double) * rank);
        or_load_row(pdtype, U, U_s, i, rank, row);
        double acc = 0.0;
        for (int k = 0; k < rank; ++k)
            acc += row[k] * t[k];
        z[i] = acc - c[i];
        mask[i] = z[i] > threshold ? 1 : 0;
        free(row);
    }
}

/* The float-format predictor (no scales). */
void or_predict(int d, int F, int rank, int pdtype, const void *V,
                const void *U, const double *c, double threshold,
                const double *x, double *t, double *z, uint8_t *mask)
{
    or_predict_q(d, F, rank, pdtype, V, NULL, U, NULL, c, threshold, x, t, z,
                 mask);
}

/* ---------------------------------------------------------------------------
 * Neuron-aware FFN over a neuron mask [PI-unite "Neuron-aware operators":
 * compute only the rows of the input matrices and the columns of the output
 * matrix that belong to active neurons, without a dense conversion;
 * PI-arch Fig. 8: inactive neurons are ignored].
 *
 *   gated (ReGLU, dReLU): g_i = Wg_i . x - c_i,  u_i = Wu_i . x
 *      ReGLU: h_i = max(g_i, 0) * u_i
 *      dReLU: h_i = max(g_i, 0) * max(u_i, 0)   [PI2-news, dReLU]
 *   non-gated (ReLU):     g_i = Wg_i . x - c_i,  h_i = max(g_i, 0)
 *   y_j = sum over i ascending with mask_i and h_i != 0 of h_i * Wdown[j, i]
 *
 * mask == NULL means every neuron (the dense FFN).  Neurons outside the mask
 * get h_i = 0.  `wdtype` gives the format of Wg, Wu and Wdown.  For float
 * formats Wdown is d x F (output-major); `down_neuron_major` = 1 means it is
 * given as its transpose F x d (the INT4 layout, where each neuron's column
 * is quantised as one vector).
 * ------------------------------------------------------------------------- */
static double or_act(int act, double g, double u)
{
    double gp = g > 0.0 ? g : 0.0;
    if (act == OR_RELU)  return gp;
    if (act == OR_REGLU) return gp * u;
    double up = u > 0.0 ? u : 0.0;             /* OR_DRELU */
    return gp * up;
}

void or_ffn_masked(int d, int F, int act, int wdtype, const void *Wg,
                   const void *Wg_s, const void *Wu, const void *Wu_s,
                   const void *Wd, const void *Wd_s, int down_neuron_major,
                   const double *c, const double *x, const uint8_t *mask,
                   double *h, double *y)
{
    #pragma omp parallel for schedule(dynamic, 16)
    for (int i = 0; i < F; ++i) {
        h[i] = 0.0;
        if (mask && !mask[i])
            continue;
        double *row = (double *)malloc(sizeof(double) * d);
        or_load_row(wdtype, Wg, Wg_s, i, d, row);
        double g = 0.0;
        for (int j = 0; j < d; ++j)
            g += row[j] * x[j];
        g -= c[i];
        double u = 0.0;
        if (act != OR_RELU) {
            or_load_row(wdtype, Wu, Wu_s, i, d, row);
            for (int j = 0; j < d; ++j)
                u += row[j] * x[j];
        }
        h[i] = or_act(act, g, u);
        free(row);
    }
    if (down_neuron_major) {
        /* Column i of Wdown is row i of the F x d transpose. */
        double *col = (double *)malloc(sizeof(double) * (size_t)d);
        for (int j = 0; j < d; ++j)
            y[j] = 0.0;
        for (int i = 0; i < F; ++i) {
            if (h[i] == 0.0)
                continue;
            or_load_row(wdtype, Wd, Wd_s, i, d, col);
            for (int j = 0; j < d; ++j)
                y[j] += h[i] * col[j];
        }
        free(col);
    } else {
        #pragma omp parallel for schedule(static)
        for (int j = 0; j < d; ++j) {
            double acc = 0.0;
            for (int i = 0; i < F; ++i) {
                if (h[i] == 0.0)
                    continue;
                acc += h[i] * or_elem(wdtype, Wd, (long)j * F + i);
            }
            y[j] = acc;
        }
    }
}

/* ---------------------------------------------------------------------------
 * MoE router (TurboSparse-Mixtral-shaped layer): logits l_e = Wr_e . x,
 * softmax over the E experts, the two largest probabilities (equal values go
 * to the lower expert index), weights renormalised over the two.  The two
 * experts are returned in ascending expert index, with their weights.
 * Wr is E x d in `rdtype`.
 * ------------------------------------------------------------------------- */
void or_route_top2(int d, int E, int rdtype, const void *Wr, const double *x,
                   double *logits, int *experts, double *weights)
{
    double *row = (double *)malloc(sizeof(double) * d);
    for (int e = 0; e < E; ++e) {
        or_load_row(rdtype, Wr, NULL, e, d, row);
        double acc = 0.0;
        for (int j = 0; j < d; ++j)
            acc += row[j] * x[j];
        logits[e] = acc;
    }
    free(row);
    double mx = logits[0];
    for (int e = 1; e < E; ++e)
        if (logits[e] > mx) mx = logits[e];
    double *p = (double *)malloc(sizeof(double) * E);
    double s = 0.0;
    for (int e = 0; e < E; ++e) {
        p[e] = exp(logits[e] - mx);
        s += p[e];
    }
    for (int e = 0; e < E; ++e)
        p[e] /= s;
    int a = 0;                                   /* largest, lowest index */
    for (int e = 1; e < E; ++e)
        if (p[e] > p[a]) a = e;
    int b = (a == 0) ? 1 : 0;                    /* second, lowest index */
    for (int e = 0; e < E; ++e)
        if (e != a && p[e] > p[b]) b = e;
    int lo = a < b ? a : b, hi = a < b ? b : a;
    experts[0] = lo;
    experts[1] = hi;
    weights[0] = p[lo] / (p[lo] + p[hi]);
    weights[1] = p[hi] / (p[lo] + p[hi]);
    free(p);
}

/* ---------------------------------------------------------------------------
 * Neuron table [PI-unite "Neuron placement and management": a table maps
 * each placed neuron to its original position in the matrix; PI2-rev and
 * PI2-news: the neuron cluster is the unit of work handed to one processor].
 *
 * perm[p] = original neuron id stored at table position p.  The F positions
 * are cut into S strips (one per processor: S = number of SMs on the GPU);
 * strip b holds n_b = floor(F/S) + (b < F mod S) neurons at positions
 * [off_b, off_b + n_b).  Neurons are ranked by descending profiled frequency
 * (equal frequencies by ascending id) and dealt like cards: round j visits the
 * strips in ascending order for even j and descending order for odd j, and
 * each visited strip that still has room takes the next-ranked neuron.  A
 * strip keeps its neurons in the order received (hottest first).  freq ==
 * NULL gives the identity table.
 * ------------------------------------------------------------------------- */
static const double *g_sort_freq;
static int or_cmp_rank(const void *pa, const void *pb)
{
    int a = *(const int *)pa, b = *(const int *)pb;
    if (g_sort_freq[a] > g_sort_freq[b]) return -1;
    if (g_sort_freq[a] < g_sort_freq[b]) return 1;
    return (a > b) - (a < b);
}

void or_strip_offsets(int F, int S, int32_t *off)
{
    int q = F / S, rem = F % S;
    off[0] = 0;
    for (int b = 0; b < S; ++b)
        off[b + 1] = off[b] + q + (b < rem ? 1 : 0);
}

void or_neuron_table(int F, int S, const double *freq, int32_t *perm)
{
    if (!freq) {
        for (int p = 0; p < F; ++p)
            perm[p] = p;
        return;
    }
    int *order = (int *)malloc(sizeof(int) * F);
    for (int i = 0; i < F; ++i)
        order[i] = i;
    g_sort_freq = freq;
    qsort(order, (size_t)F, sizeof(int), or_cmp_rank);
    int32_t *off = (int32_t *)malloc(sizeof(int32_t) * (S + 1));
    int *fill = (int *)calloc((size_t)S, sizeof(int));
    or_strip_offsets(F, S, off);
    int next = 0;
    for (int round = 0; next < F; ++round) {
        for (int k = 0; k < S && next < F; ++k) {
            int b = (round % 2 == 0) ? k : S - 1 - k;
            if (fill[b] < off[b + 1] - off[b]) {
                perm[off[b] + fill[b]] = order[next++];
                fill[b]++;
            }
        }
    }
    free(fill);
    free(off);
    free(order);
}
