/*
 * CPU oracle for the fine-grained MoE feed-forward layer.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the plain, slow, double-precision
 * statement of what the layer computes. Only the test suite, the smoke check
 * and the benchmark's CPU-baseline leg load it; the product path never does.
 * It shares no code, header or constant with the CUDA library.
 *
 * Sources (all on the page "Inside Kolibri 1: Hybrid RNoPE Attention, Sparse
 * MoE, and FP8 Serving", flozi.net, unless noted):
 *   - section "Routing: selection bias and mixture weights are separate":
 *       router gives FP32 logits [N, 384] from x [N, 2560]; the learned
 *       correction bias is added to the logits only to pick the top six;
 *       the mixture weights are sigmoid of the UNBIASED logits of those six,
 *       not renormalised; each expert (routed or shared) is a SwiGLU MLP,
 *       SiLU(gate) x up followed by the down projection, no biases; one
 *       shared expert is always on in addition to the six routed ones.
 *   - section "The FP8 path is explicitly mixed precision": E4M3 weights in
 *       128 x 128 blocks with one FP32 scale per block.
 *   - page "Kolibri 1 Deep Dive" (abrarakhunji.com), section 1, "Mathematical
 *       Routing & Load Balancing Formulation": the layer output is the
 *       gate-weighted sum of the selected experts' SwiGLU outputs (the
 *       residual "x +" of that formula lies outside this layer).
 *
 * Readings where the pages leave a step open:
 *   - ties in the biased score go to the lower expert index; the six chosen
 *     experts are listed by biased score, highest first;
 *   - the shared expert enters the sum with weight 1;
 *   - the dispatch order groups the (token, slot) pairs by expert, ascending,
 *     and by token, ascending, inside one expert (a counting sort);
 *   - inputs are read exactly as stored (BF16 and FP32 widened to double,
 *     E4M3 decoded from its bits and multiplied by its FP32 block scale),
 *     and every sum runs in index order, in double.
 *
 * Parity pins: every function here is pinned by the CPU tests in
 * tests/test_oracle.py (brute-force top-k, library sort, numpy float64
 * matmul, the 256 E4M3 codes and the E4M3 encoder against torch, closed
 * forms and hand-computed cases).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* dtype codes used by the oracle's own entry points */
enum { OR_F32 = 0, OR_BF16 = 1, OR_E4M3 = 2 };

#define OR_BLOCK 128

static double bf16_bits_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP 8-bit float E4M3 ("fn" flavour): sign, 4 exponent bits with bias 7,
 * 3 mantissa bits; exponent field 0 holds subnormals m/8 * 2^-6; there are no
 * infinities; the two codes with all exponent and mantissa bits set are NaN. */
double oracle_e4m3_to_double(uint8_t q)
{
    int sign = q >> 7;
    int ex = (q >> 3) & 15;
    int man = q & 7;
    double v;
    if (ex == 15 && man == 7)
        return NAN;
    if (ex == 0)
        v = ldexp((double)man / 8.0, -6);
    else
        v = ldexp(1.0 + (double)man / 8.0, ex - 7);
    return sign ? -v : v;
}

/* Element (r, c) of matrix `m` (rows x cols, row-major) of expert `g` in a
 * stacked weight tensor [G, rows, cols]; E4M3 values carry the FP32 scale of
 * their 128 x 128 block, stored as [G, rows/128, cols/128]. */
static double weight_at(const void *w, const float *scale, int dtype,
                        int64_t g, int rows, int cols, int r, int c)
{
    int64_t i = (g * rows + r) * (int64_t)cols + c;
    switch (dtype) {
    case OR_F32:
        return (double)((const float *)w)[i];
    case OR_BF16:
        return bf16_bits_to_double(((const uint16_t *)w)[i]);
    default: {
        int rb = rows / OR_BLOCK, cb = cols / OR_BLOCK;
        double s = (double)scale[(g * rb + r / OR_BLOCK) * (int64_t)cb + c / OR_BLOCK];
        return oracle_e4m3_to_double(((const uint8_t *)w)[i]) * s;
    }
    }
}

static double input_at(const void *x, int dtype, int64_t i)
{
    return dtype == OR_F32 ? (double)((const float *)x)[i]
                           : bf16_bits_to_double(((const uint16_t *)x)[i]);
}

/* Router: l[t][e] = sum_j x[t][j] * W_r[e][j], summed in j order.
 * x is [N, d] (FP32 or BF16), W_r is [E, d] FP32, logits are [N, E]. */
void oracle_router_logits(int N, int d, int E, const void *x, int x_dtype,
                          const float *w_router, double *logits, int nthreads)
{
    int t;
#pragma omp parallel for num_threads(nthreads) schedule(static)
    for (t = 0; t < N; ++t) {
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int j = 0; j < d; ++j)
                acc += input_at(x, x_dtype, (int64_t)t * d + j) * (double)w_router[(int64_t)e * d + j];
            logits[(int64_t)t * E + e] = acc;
        }
    }
}

static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

/* Selection and mixture weights for every token:
 *   s[e] = l[e] + b[e];
 *   idx  = the first K experts of 0..E-1 ordered by (s descending, e ascending);
 *   score 0 ("Inside Kolibri 1", routing section):
 *     g[k] = sigmoid(l[idx[k]])   (unbiased logit, no renormalisation);
 *   score 1 ("Kolibri 1 Deep Dive", "Mathematical Routing & Load Balancing
 *   Formulation": a softmax over the selected experts' logits):
 *     g[k] = exp(l[idx[k]]) / sum_j exp(l[idx[j]])   (unbiased logits;
 *     evaluated with the largest selected logit subtracted first);
 *   margin = s of the K-th choice minus s of the (K+1)-th (HUGE_VAL if E == K).
 * K passes of "take the best remaining" give exactly that ordered prefix. */
void oracle_select_score(int N, int E, int K, const double *logits, const float *bias, int score,
                         int32_t *idx, double *g, double *margin)
{
    unsigned char *taken = (unsigned char *)malloc((size_t)E);
    for (int t = 0; t < N; ++t) {
        const double *l = logits + (int64_t)t * E;
        memset(taken, 0, (size_t)E);
        double last = 0.0;
        for (int k = 0; k <= K && k < E; ++k) {
            int best = -1;
            double best_s = 0.0;
            for (int e = 0; e < E; ++e) {
                if (taken[e])
                    continue;
                double s = l[e] + (double)bias[e];
                if (best < 0 || s > best_s) {   /* strict: equal s keeps the lower e */
                    best = e;
                    best_s = s;
                }
            }
            taken[best] = 1;
            if (k < K) {
                idx[(int64_t)t * K + k] = best;
                g[(int64_t)t * K + k] = sigmoid(l[best]);
                last = best_s;
            } else {
                margin[t] = last - best_s;
            }
        }
        if (E == K)
            margin[t] = HUGE_VAL;
        if (score == 1) {
            double *gt = g + (int64_t)t * K, mx = -HUGE_VAL, sum = 0.0;
            for (int k = 0; k < K; ++k)
                mx = fmax(mx, l[idx[(int64_t)t * K + k]]);
            for (int k = 0; k < K; ++k) {
                gt[k] = exp(l[idx[(int64_t)t * K + k]] - mx);
                sum += gt[k];
            }
            for (int k = 0; k < K; ++k)
                gt[k] /= sum;
        }
    }
    free(taken);
}

void oracle_select(int N, int E, int K, const double *logits, const float *bias,
                   int32_t *idx, double *g, double *margin)
{
    oracle_select_score(N, E, K, logits, bias, 0, idx, g, margin);
}

/* Dispatch by counting sort.
 *   counts[e]   = number of (t, k) with idx[t][k] == e
 *   offsets     = exclusive prefix sum of counts, offsets[E] = N*K
 *   perm_token  = token of each dispatched row, rows grouped by expert
 *                 ascending and, inside one expert, by token ascending
 *   inv_pos[t][k] = the dispatched row that holds (t, k)
 * Returns 0, or -1 when an index lies outside 0..E-1. */
int oracle_permute(int N, int K, int E, const int32_t *idx, int32_t *counts,
                   int32_t *offsets, int32_t *perm_token, int32_t *inv_pos)
{
    int32_t *fill = (int32_t *)calloc((size_t)E, sizeof(int32_t));
    memset(counts, 0, (size_t)E * sizeof(int32_t));
    for (int64_t i = 0; i < (int64_t)N * K; ++i) {
        if (idx[i] < 0 || idx[i] >= E) {
            free(fill);
            return -1;
        }
        counts[idx[i]]++;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e)
        offsets[e + 1] = offsets[e] + counts[e];
    for (int t = 0; t < N; ++t) {
        for (int k = 0; k < K; ++k) {
            int e = idx[(int64_t)t * K + k];
            int32_t pos = offsets[e] + fill[e]++;
            perm_token[pos] = t;
            inv_pos[(int64_t)t * K + k] = pos;
        }
    }
    free(fill);
    return 0;
}

/* One SwiGLU expert on one token: out = W_d (SiLU(W_g x) * (W_u x)).
 * W_g, W_u are [I, d] and W_d is [d, I] inside stacked [G, ., .] tensors;
 * SiLU(z) = z / (1 + exp(-z)). `h` is caller scratch of I doubles. */
static void expert_ffn(int d, int I, const double *xrow, int64_t g, int w_dtype,
                       const void *wg, const void *wu, const void *wd,
                       const float *sg, const float *su, const float *sd,
                       double *h, double *out)
{
    for (int i = 0; i < I; ++i) {
        double a = 0.0, b = 0.0;
        for (int j = 0; j < d; ++j) {
            a += weight_at(wg, sg, w_dtype, g, I, d, i, j) * xrow[j];
            b += weight_at(wu, su, w_dtype, g, I, d, i, j) * xrow[j];
        }
        h[i] = a * sigmoid(a) * b;
    }
    for (int j = 0; j < d; ++j) {
        double acc = 0.0;
        for (int i = 0; i < I; ++i)
            acc += weight_at(wd, sd, w_dtype, g, d, I, j, i) * h[i];
        out[j] = acc;
    }
}

/* F_g(x_t) for a list of (token, expert) pairs: out is [n_pairs, d].
 * x is [N, d]; expert g indexes the stacked [G, ., .] tensors. */
void oracle_expert_outputs(int d, int I, const void *x, int x_dtype, int w_dtype,
                           const void *wg, const void *wu, const void *wd,
                           const float *sg, const float *su, const float *sd,
                           int n_pairs, const int32_t *tokens, const int32_t *experts,
                           double *out, int nthreads)
{
    int p;
#pragma omp parallel for num_threads(nthreads) schedule(dynamic)
    for (p = 0; p < n_pairs; ++p) {
        double *xrow = (double *)malloc((size_t)d * sizeof(double));
        double *h = (double *)malloc((size_t)I * sizeof(double));
        for (int j = 0; j < d; ++j)
            xrow[j] = input_at(x, x_dtype, (int64_t)tokens[p] * d + j);
        expert_ffn(d, I, xrow, experts[p], w_dtype, wg, wu, wd, sg, su, sd, h,
                   out + (int64_t)p * d);
        free(h);
        free(xrow);
    }
}

/* The whole layer for a chosen subset of tokens (rows[0..n_rows-1] index x):
 *   y[t] = F_shared(x[t]) + sum_{k<K} g[t][k] * F_{idx[t][k]}(x[t])
 * with the shared expert stored at index E of the stacked weight tensors.
 * Writes y [n_rows, d], and the selection idx/g [n_rows, K] and margin
 * [n_rows] of those tokens. */
void oracle_layer_score(int N, int d, int E, int K, int I,
                        const void *x, int x_dtype, const float *w_router, const float *bias,
                        const void *wg, const void *wu, const void *wd,
                        const float *sg, const float *su, const float *sd, int w_dtype,
                        int n_rows, const int32_t *rows, int score,
                        double *y, int32_t *idx_out, double *g_out, double *margin_out,
                        int nthreads)
{
    int r;
    (void)N;
#pragma omp parallel for num_threads(nthreads) schedule(dynamic)
    for (r = 0; r < n_rows; ++r) {
        int64_t t = rows[r];
        double *xrow = (double *)malloc((size_t)d * sizeof(double));
        double *l = (double *)malloc((size_t)E * sizeof(double));
        double *h = (double *)malloc((size_t)I * sizeof(double));
        double *f = (double *)malloc((size_t)d * sizeof(double));
        double *yr = y + (int64_t)r * d;
        for (int j = 0; j < d; ++j)
            xrow[j] = input_at(x, x_dtype, t * d + j);
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int j = 0; j < d; ++j)
                acc += xrow[j] * (double)w_router[(int64_t)e * d + j];
            l[e] = acc;
        }
        oracle_select_score(1, E, K, l, bias, score, idx_out + (int64_t)r * K, g_out + (int64_t)r * K,
                            margin_out + r);
        expert_ffn(d, I, xrow, E, w_dtype, wg, wu, wd, sg, su, sd, h, yr);
        for (int k = 0; k < K; ++k) {
            int e = idx_out[(int64_t)r * K + k];
            double gk = g_out[(int64_t)r * K + k];
            expert_ffn(d, I, xrow, e, w_dtype, wg, wu, wd, sg, su, sd, h, f);
            for (int j = 0; j < d; ++j)
                yr[j] += gk * f[j];
        }
        free(f);
        free(h);
        free(l);
        free(xrow);
    }
}

void oracle_layer(int N, int d, int E, int K, int I,
                  const void *x, int x_dtype, const float *w_router, const float *bias,
                  const void *wg, const void *wu, const void *wd,
                  const float *sg, const float *su, const float *sd, int w_dtype,
                  int n_rows, const int32_t *rows,
                  double *y, int32_t *idx_out, double *g_out, double *margin_out,
                  int nthreads)
{
    oracle_layer_score(N, d, E, K, I, x, x_dtype, w_router, bias, wg, wu, wd, sg, su, sd, w_dtype, n_rows, rows, 0,
                       y, idx_out, g_out, margin_out, nthreads);
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------
 * Sandwich block around the MoE sublayer ("Inside Kolibri 1", section "The
 * released stack": RMSNorm before and after the MoE, a residual addition
 * after it). The pages give no epsilon; it is an argument.
 *   x     = bf16( h / sqrt(mean_j h_j^2 + eps) * g_pre )
 *   m     = the MoE layer on x (oracle_layer_score, in double)
 *   h_out = h + m / sqrt(mean_j m_j^2 + eps) * g_post     (in double)
 * The layer input x is stored in BF16, as the CUDA path stores it, so that
 * the top-K is decided on the same input; bf16() rounds to nearest, ties to
 * even, directly from double.
 * ---------------------------------------------------------------------- */
static uint16_t double_to_bf16_rne(double v)
{
    if (v == 0.0 || !isfinite(v)) {
        float f = (float)v;
        uint32_t u;
        memcpy(&u, &f, 4);
        return (uint16_t)(u >> 16);
    }
    int e;
    frexp(v, &e);                                    /* v = f * 2^e, 0.5 <= |f| < 1 */
    const double q = ldexp(nearbyint(ldexp(v, 8 - e)), e - 8);   /* 8 significant bits, ties to even */
    const float f = (float)q;                        /* exact: q has 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

/* x[t] = bf16(h[t] / sqrt(mean(h[t]^2) + eps) * gamma) for N rows of BF16 h. */
void oracle_rmsnorm_bf16(int N, int d, const uint16_t *h, const uint16_t *gamma, double eps, uint16_t *x)
{
    for (int64_t t = 0; t < N; ++t) {
        double ss = 0.0;
        for (int j = 0; j < d; ++j) {
            const double v = bf16_bits_to_double(h[t * d + j]);
            ss += v * v;
        }
        const double r = 1.0 / sqrt(ss / d + eps);
        for (int j = 0; j < d; ++j)
            x[t * d + j] = double_to_bf16_rne(bf16_bits_to_double(h[t * d + j]) * r * bf16_bits_to_double(gamma[j]));
    }
}

/* h_out[r] = h[rows[r]] + m[r] / sqrt(mean(m[r]^2) + eps) * g_post, with m the
 * MoE output rows already computed (oracle_layer_score on the normalised x). */
void oracle_post_residual(int N, int d, int n_rows, const int32_t *rows, const uint16_t *h, const double *m,
                          const uint16_t *g_post, double eps, double *h_out)
{
    (void)N;
    for (int64_t r = 0; r < n_rows; ++r) {
        double ss = 0.0;
        for (int j = 0; j < d; ++j)
            ss += m[r * d + j] * m[r * d + j];
        const double s = 1.0 / sqrt(ss / d + eps);
        for (int j = 0; j < d; ++j)
            h_out[r * d + j] = bf16_bits_to_double(h[(int64_t)rows[r] * d + j]) + m[r * d + j] * s *
                               bf16_bits_to_double(g_post[j]);
    }
}

/* ----------------------------------------------------------------------
 * FP8 activations ("Inside Kolibri 1", section "The FP8 path is explicitly
 * mixed precision": activations are quantised dynamically in groups of
 * 1 x 128; the weights are E4M3 in 128 x 128 blocks with FP32 scales).
 *
 * Readings where the page is silent:
 *   - a group is 128 consecutive columns of one row of a GEMM input (x for
 *     the gate and up projections, H for the down projection);
 *   - its scale is s = amax / 448 in FP32 (448 = the largest E4M3 value),
 *     s = 1 for an all-zero group, used as computed (never rounded to 2^k,
 *     like the weight scales);
 *   - a code is E4M3(v), v = x / s computed in FP32, rounded to nearest with
 *     ties to even and saturated to +-448; the code decision is taken in
 *     FP32, the precision a kernel computes it in;
 *   - H is rounded to BF16 before it is quantised, as the layer stores H;
 *   - the GEMMs are exact: for each 128-column block kb,
 *       out += s_act[kb] * s_w[kb] * sum_k E4M3(q_act[k]) * E4M3(q_w[k]),
 *     summed in index order in double.
 * ---------------------------------------------------------------------- */

/* E4M3 code of a finite float: round to nearest, ties to even, saturate to
 * +-448. Codes: sign bit 7, exponent bits 6..3 (bias 7; 0 = subnormal),
 * mantissa bits 2..0; subnormals are m * 2^-9. */
uint8_t oracle_float_to_e4m3(float v)
{
    const uint8_t sign = signbit(v) ? 0x80 : 0x00;
    const double a = fabs((double)v);
    if (a == 0.0) return sign;
    if (a < ldexp(1.0, -6)) {                          /* below the smallest normal: quantum 2^-9 */
        const double m = nearbyint(ldexp(a, 9));       /* 0 .. 8; 8 is the smallest normal 2^-6 */
        return (uint8_t)(sign | (uint8_t)m);
    }
    int e;
    frexp(a, &e);                                      /* a = f * 2^e, 0.5 <= f < 1: a in [2^(e-1), 2^e) */
    int ex = e - 1;                                    /* unbiased exponent, ex >= -6 */
    double m = nearbyint(ldexp(a, 3 - ex));            /* significand in eighths: 8 .. 16 */
    if (m == 16.0) {
        m = 8.0;
        ex += 1;
    }
    if (ex > 8 || (ex == 8 && m > 14.0)) return (uint8_t)(sign | 0x7E);   /* saturate: 1.75 * 2^8 = 448 */
    return (uint8_t)(sign | (uint8_t)((ex + 7) << 3) | (uint8_t)(m - 8.0));
}

/* Quantises `rows` rows of `cols` BF16 values in groups of 128 columns:
 * codes [rows, cols], scales [rows, cols / 128]. */
void oracle_quant_1x128(int rows, int cols, const uint16_t *x, uint8_t *codes, float *scales)
{
    const int groups = cols / OR_BLOCK;
    for (int r = 0; r < rows; ++r)
        for (int g = 0; g < groups; ++g) {
            const int64_t base = (int64_t)r * cols + (int64_t)g * OR_BLOCK;
            float amax = 0.0f;
            for (int k = 0; k < OR_BLOCK; ++k) {
                const float v = fabsf((float)bf16_bits_to_double(x[base + k]));
                if (v > amax) amax = v;
            }
            const float s = amax > 0.0f ? amax / 448.0f : 1.0f;
            scales[(int64_t)r * groups + g] = s;
            for (int k = 0; k < OR_BLOCK; ++k)
                codes[base + k] = oracle_float_to_e4m3((float)bf16_bits_to_double(x[base + k]) / s);
        }
}

/* One SwiGLU expert `g` (E4M3 weights) on one token whose row is quantised:
 * xq [d] codes with xs [d / 128] scales. H is formed in double, rounded to
 * BF16, quantised in 1 x 128 groups, and the down projection runs on those
 * codes. `hb` (I BF16), `hq` (I codes), `hs` (I / 128 scales) are scratch. */
static void expert_ffn_a8(int d, int I, const uint8_t *xq, const float *xs, int64_t g,
                          const uint8_t *wg, const uint8_t *wu, const uint8_t *wd,
                          const float *sg, const float *su, const float *sd,
                          uint16_t *hb, uint8_t *hq, float *hs, double *out)
{
    const int db = d / OR_BLOCK, ib = I / OR_BLOCK;
    for (int i = 0; i < I; ++i) {
        double a = 0.0, b = 0.0;
        for (int kb = 0; kb < db; ++kb) {
            double pa = 0.0, pb = 0.0;
            for (int k = kb * OR_BLOCK; k < (kb + 1) * OR_BLOCK; ++k) {
                const double xv = oracle_e4m3_to_double(xq[k]);
                const int64_t wi = (g * I + i) * (int64_t)d + k;
                pa += xv * oracle_e4m3_to_double(wg[wi]);
                pb += xv * oracle_e4m3_to_double(wu[wi]);
            }
            const int64_t si = (g * ib + i / OR_BLOCK) * (int64_t)db + kb;
            a += (double)xs[kb] * (double)sg[si] * pa;
            b += (double)xs[kb] * (double)su[si] * pb;
        }
        hb[i] = double_to_bf16_rne(a * sigmoid(a) * b);
    }
    oracle_quant_1x128(1, I, hb, hq, hs);
    for (int j = 0; j < d; ++j) {
        double acc = 0.0;
        for (int kb = 0; kb < ib; ++kb) {
            double p = 0.0;
            for (int k = kb * OR_BLOCK; k < (kb + 1) * OR_BLOCK; ++k)
                p += oracle_e4m3_to_double(hq[k]) * oracle_e4m3_to_double(wd[(g * d + j) * (int64_t)I + k]);
            acc += (double)hs[kb] * (double)sd[(g * db + j / OR_BLOCK) * (int64_t)ib + kb] * p;
        }
        out[j] = acc;
    }
}

/* F_g(x_t) with FP8 activations for a list of (token, expert) pairs: the
 * token's row is quantised in 1 x 128 groups and expert_ffn_a8 runs on it.
 * x is [N, d] BF16; out is [n_pairs, d]; expert g indexes the stacked
 * [G, ., .] E4M3 tensors. */
void oracle_expert_outputs_a8(int d, int I, const uint16_t *x,
                              const uint8_t *wg, const uint8_t *wu, const uint8_t *wd,
                              const float *sg, const float *su, const float *sd,
                              int n_pairs, const int32_t *tokens, const int32_t *experts,
                              double *out, int nthreads)
{
    int p;
#pragma omp parallel for num_threads(nthreads) schedule(dynamic)
    for (p = 0; p < n_pairs; ++p) {
        uint8_t *xq = (uint8_t *)malloc((size_t)d);
        float *xs = (float *)malloc((size_t)(d / OR_BLOCK) * sizeof(float));
        uint16_t *hb = (uint16_t *)malloc((size_t)I * sizeof(uint16_t));
        uint8_t *hq = (uint8_t *)malloc((size_t)I);
        float *hs = (float *)malloc((size_t)(I / OR_BLOCK) * sizeof(float));
        oracle_quant_1x128(1, d, x + (int64_t)tokens[p] * d, xq, xs);
        expert_ffn_a8(d, I, xq, xs, experts[p], wg, wu, wd, sg, su, sd, hb, hq, hs, out + (int64_t)p * d);
        free(hs);
        free(hq);
        free(hb);
        free(xs);
        free(xq);
    }
}

/* The whole layer with FP8 activations, for tokens rows[0 .. n_rows-1]:
 * the router and the top-K see x as stored (BF16); each expert sees x
 * quantised in 1 x 128 groups, and its down projection sees H quantised the
 * same way. E4M3 weights only. Outputs as oracle_layer_score. */
void oracle_layer_a8(int N, int d, int E, int K, int I,
                     const uint16_t *x, const float *w_router, const float *bias,
                     const uint8_t *wg, const uint8_t *wu, const uint8_t *wd,
                     const float *sg, const float *su, const float *sd,
                     int n_rows, const int32_t *rows, int score,
                     double *y, int32_t *idx_out, double *g_out, double *margin_out, int nthreads)
{
    int r;
    (void)N;
#pragma omp parallel for num_threads(nthreads) schedule(dynamic)
    for (r = 0; r < n_rows; ++r) {
        const int64_t t = rows[r];
        double *l = (double *)malloc((size_t)E * sizeof(double));
        double *f = (double *)malloc((size_t)d * sizeof(double));
        uint8_t *xq = (uint8_t *)malloc((size_t)d);
        float *xs = (float *)malloc((size_t)(d / OR_BLOCK) * sizeof(float));
        uint16_t *hb = (uint16_t *)malloc((size_t)I * sizeof(uint16_t));
        uint8_t *hq = (uint8_t *)malloc((size_t)I);
        float *hs = (float *)malloc((size_t)(I / OR_BLOCK) * sizeof(float));
        double *yr = y + (int64_t)r * d;
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int j = 0; j < d; ++j)
                acc += bf16_bits_to_double(x[t * d + j]) * (double)w_router[(int64_t)e * d + j];
            l[e] = acc;
        }
        oracle_select_score(1, E, K, l, bias, score, idx_out + (int64_t)r * K, g_out + (int64_t)r * K,
                            margin_out + r);
        oracle_quant_1x128(1, d, x + t * d, xq, xs);
        expert_ffn_a8(d, I, xq, xs, E, wg, wu, wd, sg, su, sd, hb, hq, hs, yr);
        for (int k = 0; k < K; ++k) {
            const int e = idx_out[(int64_t)r * K + k];
            const double gk = g_out[(int64_t)r * K + k];
            expert_ffn_a8(d, I, xq, xs, e, wg, wu, wd, sg, su, sd, hb, hq, hs, f);
            for (int j = 0; j < d; ++j)
                yr[j] += gk * f[j];
        }
        free(hs);
        free(hq);
        free(hb);
        free(xs);
        free(xq);
        free(f);
        free(l);
    }
}
