/*
 * prox_oracle.c -- plain, slow, fp64 CPU oracle of the Prox two-stage sparse
 * SwiGLU FFN.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark load this file's library. It shares no code, header,
 * table or constant with the CUDA library: it is written from the method's
 * definitions, one step at a time, with no blocking, fusion or reordering.
 *
 * Sources (all are pages about "Prox: Training-Free FFN Activation Sparsity
 * via Approximate Intermediate-Channel Salience in LLMs"):
 *   [blog]  the Prox deep-dive blog post ("Prox 完全拆解"), its sections
 *           "Why the SwiGLU intermediate state", "Stage 1", "Stage 2",
 *           "Compute budget" and "From formula to GPU";
 *   [arxiv] the translated arXiv HTML, section 2.1 (SwiGLU FFN definition)
 *           and section 2.2 (input-sparse and output-sparse projections).
 *
 * Storage formats (the library's formats, restated here independently):
 *   bf16 values are uint16 bit patterns (the upper half of an IEEE binary32);
 *   w_up_cm, w_gate_cm : [d_ff][d_model], channel j is row j (W_up[:, j]);
 *   w_down             : [d_ff][d_model], row j is W_down[j, :];
 *   proxy q            : [d_model][d_ff/2] bytes, row i holds W~[i, :],
 *                        channel 2m in the low nibble of byte m, 2m+1 in the
 *                        high nibble, two's complement;
 *   proxy scale        : [d_model] fp32, one per row i of W (d_model x d_ff).
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fopenmp -shared.
 * The fp32 steps of the quantiser (scale = max/7, W/scale, round half to
 * even) rely on IEEE single-precision division, which that build gives.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_value(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static float bf16_value_f(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* SiLU(z) = z * sigmoid(z) = z / (1 + exp(-z))   [arxiv 2.1; blog "Why s"] */
static double silu(double z)
{
    return z / (1.0 + exp(-z));
}

/* GELU(z) = z * Phi(z) = z (1 + erf(z / sqrt 2)) / 2, the gate activation of
 * the GeGLU-style models the pages also evaluate [blog "Evidence"]. Reading
 * adopted: the exact (erf) GELU; the pages do not name a variant. */
static double gelu(double z)
{
    return 0.5 * z * (1.0 + erf(z / sqrt(2.0)));
}

/* act 0: SwiGLU (SiLU gate), act 1: GeGLU (GELU gate) */
static double activation(double z, int act)
{
    return act == 1 ? gelu(z) : silu(z);
}

/* ------------------------------------------------------------------------
 * Offline: symmetric per-row INT4 proxy copy of one projection
 * [blog "Stage 1": W~_up and W~_gate are symmetric per-row INT4 copies].
 *
 * Reading adopted: "row" is a row i of W in the pages' own orientation
 * W in R^{d_model x d_ff} (one scale per input coordinate), so that the
 * input-sparse proxy product skips whole rows. Symmetric range [-7, 7],
 * scale = max_j |W[i,j]| / 7 in fp32, q = clamp(round_half_even(W/scale)),
 * all-zero row -> scale 0, q 0.
 * ---------------------------------------------------------------------- */
void oracle_quantize_proxy(int d_model, int d_ff, const uint16_t *w_cm,
                           uint8_t *q, float *scale)
{
    if (d_model <= 0 || d_ff <= 1)
        return;
    const size_t half = (size_t)(d_ff / 2);
    for (int i = 0; i < d_model; ++i) {
        float amax = 0.0f;
        for (int j = 0; j < d_ff; ++j) {
            float a = fabsf(bf16_value_f(w_cm[(size_t)j * d_model + i]));
            if (a > amax)
                amax = a;
        }
        float s = amax / 7.0f;
        scale[i] = s;
        uint8_t *row = q + (size_t)i * half;
        memset(row, 0, half);
        for (int j = 0; j < d_ff; ++j) {
            int v = 0;
            if (s > 0.0f) {
                float r = bf16_value_f(w_cm[(size_t)j * d_model + i]) / s;
                v = (int)nearbyintf(r);
                if (v > 7) v = 7;
                if (v < -7) v = -7;
            }
            uint8_t nib = (uint8_t)(v & 0xF);
            if (j % 2 == 0)
                row[j / 2] |= nib;
            else
                row[j / 2] |= (uint8_t)(nib << 4);
        }
    }
}

/* Dequantised proxy weight W~[i, j] = scale_i * q_ij (exact in fp64). */
static double proxy_weight(const uint8_t *q, const float *scale, int d_ff,
                           int i, int j)
{
    uint8_t byte = q[(size_t)i * (d_ff / 2) + j / 2];
    int nib = (j % 2 == 0) ? (byte & 0xF) : (byte >> 4);
    int v = (nib >= 8) ? nib - 16 : nib;
    return (double)scale[i] * (double)v;
}

/* ------------------------------------------------------------------------
 * Stage 1 for one token [blog "Stage 1"]:
 *   [m_x]_i = 1[|x_i| >= tau_x]
 *   u~ = Pi_in(x, W~_up, m_x),  h~ = SiLU(Pi_in(x, W~_gate, m_x))
 *   s~ = u~ (.) h~,             [m_s]_j = 1[|s~_j| >= tau_s]
 * with Pi_in(x, W, m) = x_[I(m)] W_[I(m), :]   [arxiv 2.2].
 * x enters unquantised; only the weights are INT4. With pw_up and pw_gate
 * given (bf16 [d_ff][d_model], the original weights) the proxy is that bf16
 * weight instead of the INT4 copy: the FP16/bf16-proxy ablation of the blog's
 * "Evidence" section (q and scale are then ignored).
 * Outputs: mask_x[d_model], u_proxy/g_proxy/s_proxy[d_ff] (g is the
 * pre-activation proxy gate), mask_s[d_ff]. Any output may be NULL.
 * ---------------------------------------------------------------------- */
void oracle_stage1_token(int d_model, int d_ff, const uint16_t *x, float tau_x,
                         const uint8_t *q_up, const float *s_up,
                         const uint8_t *q_gate, const float *s_gate,
                         float tau_s, uint8_t *mask_x, double *u_proxy,
                         double *g_proxy, double *s_proxy, uint8_t *mask_s, int act,
                         const uint16_t *pw_up, const uint16_t *pw_gate)
{
    uint8_t *mx = (uint8_t *)malloc((size_t)d_model);
    for (int i = 0; i < d_model; ++i)
        mx[i] = fabs(bf16_value(x[i])) >= (double)tau_x;
    if (mask_x)
        memcpy(mask_x, mx, (size_t)d_model);

    /* Row-outer loop: every channel still sums its terms in ascending i. */
    double *u = (double *)calloc((size_t)d_ff, sizeof(double));
    double *g = (double *)calloc((size_t)d_ff, sizeof(double));
    for (int i = 0; i < d_model; ++i) {
        if (!mx[i])
            continue;
        double xi = bf16_value(x[i]);
        for (int j = 0; j < d_ff; ++j) {
            u[j] += xi * (pw_up ? bf16_value(pw_up[(size_t)j * d_model + i])
                                : proxy_weight(q_up, s_up, d_ff, i, j));
            g[j] += xi * (pw_gate ? bf16_value(pw_gate[(size_t)j * d_model + i])
                                  : proxy_weight(q_gate, s_gate, d_ff, i, j));
        }
    }
    for (int j = 0; j < d_ff; ++j) {
        double s = u[j] * activation(g[j], act);
        if (u_proxy) u_proxy[j] = u[j];
        if (g_proxy) g_proxy[j] = g[j];
        if (s_proxy) s_proxy[j] = s;
        if (mask_s) mask_s[j] = fabs(s) >= (double)tau_s;
    }
    free(u);
    free(g);
    free(mx);
}

/* ------------------------------------------------------------------------
 * Stage 2 for one token, given the channel mask m_s [blog "Stage 2"]:
 *   u_sp = Pi_out(x, W_up, m_s),  h_sp = SiLU(Pi_out(x, W_gate, m_s))
 *   s_sp = u_sp (.) h_sp,         y = Pi_in(s_sp, W_down, m_s)
 * with Pi_out(x, W, m) = x W_[:, I(m)]   [arxiv 2.2].
 * Uses the original bf16 weights and the full (unmasked) x.
 * s_exact[d_ff] (zero on dropped channels) and y[d_model] are fp64.
 * ---------------------------------------------------------------------- */
void oracle_stage2_token(int d_model, int d_ff, const uint16_t *x,
                         const uint16_t *w_up_cm, const uint16_t *w_gate_cm,
                         const uint16_t *w_down, const uint8_t *mask_s,
                         double *s_exact, double *y, int act)
{
    for (int k = 0; k < d_model; ++k)
        y[k] = 0.0;
    for (int j = 0; j < d_ff; ++j) {
        double s = 0.0;
        if (mask_s[j]) {
            double u = 0.0, g = 0.0;
            for (int i = 0; i < d_model; ++i) {
                double xi = bf16_value(x[i]);
                u += xi * bf16_value(w_up_cm[(size_t)j * d_model + i]);
                g += xi * bf16_value(w_gate_cm[(size_t)j * d_model + i]);
            }
            s = u * activation(g, act);
            for (int k = 0; k < d_model; ++k)
                y[k] += s * bf16_value(w_down[(size_t)j * d_model + k]);
        }
        if (s_exact)
            s_exact[j] = s;
    }
}

/* ------------------------------------------------------------------------
 * Whole forward over a batch of tokens, each with its own masks (the
 * thresholds are per-layer scalars shared by all tokens and channels).
 * Tokens are independent, so they are spread over OpenMP threads; each
 * token's arithmetic is the sequential code above, so results do not depend
 * on the thread count. If mask_s_in is non-NULL it replaces the oracle's own
 * Stage-1 channel mask in Stage 2 (used to score a device mask).
 * Returns the number of threads used.
 * ---------------------------------------------------------------------- */
int oracle_forward(int d_model, int d_ff, int batch, const uint16_t *x,
                   float tau_x, float tau_s,
                   const uint16_t *w_up_cm, const uint16_t *w_gate_cm,
                   const uint16_t *w_down, const uint8_t *q_up,
                   const float *s_up, const uint8_t *q_gate,
                   const float *s_gate, const uint8_t *mask_s_in,
                   uint8_t *mask_x, uint8_t *mask_s, double *s_proxy,
                   double *s_exact, double *y, int n_threads, int act,
                   const uint16_t *pw_up, const uint16_t *pw_gate)
{
    int used = 1;
#ifdef _OPENMP
    if (n_threads <= 0)
        n_threads = omp_get_max_threads();
#pragma omp parallel num_threads(n_threads)
    {
#pragma omp single
        used = omp_get_num_threads();
#pragma omp for schedule(dynamic, 1)
#else
    (void)n_threads;
    {
#endif
        for (int t = 0; t < batch; ++t) {
            const uint16_t *xt = x + (size_t)t * d_model;
            uint8_t *ms = mask_s ? mask_s + (size_t)t * d_ff
                                 : (uint8_t *)malloc((size_t)d_ff);
            oracle_stage1_token(d_model, d_ff, xt, tau_x, q_up, s_up, q_gate,
                                s_gate, tau_s,
                                mask_x ? mask_x + (size_t)t * d_model : NULL,
                                NULL, NULL,
                                s_proxy ? s_proxy + (size_t)t * d_ff : NULL, ms, act,
                                pw_up, pw_gate);
            const uint8_t *use = mask_s_in ? mask_s_in + (size_t)t * d_ff : ms;
            oracle_stage2_token(d_model, d_ff, xt, w_up_cm, w_gate_cm, w_down,
                                use,
                                s_exact ? s_exact + (size_t)t * d_ff : NULL,
                                y + (size_t)t * d_model, act);
            if (!mask_s)
                free(ms);
        }
    }
    return used;
}

/* ------------------------------------------------------------------------
 * Offline calibration of the per-layer thresholds [blog "Stage 1" (tau_x and
 * tau_s are offline per-layer thresholds) and "Evidence" (thresholds come
 * from calibration activations, per layer)].
 *
 * Reading adopted: tau = the exact order statistic of the pooled magnitudes.
 * With n pooled values sorted ascending as v[0..n-1],
 *   rank = floor((1 - keep) * n) in IEEE double (keep is a double),
 *          clamped to [0, n - 1],
 *   tau  = (float) v[rank].
 * tau_x pools |x_i| over every calibration vector and coordinate; tau_s pools
 * |s~_j| over every calibration vector and channel, with s~ computed by
 * Stage 1 at the tau_x just chosen.
 * ---------------------------------------------------------------------- */
static int cmp_double(const void *a, const void *b)
{
    double x = *(const double *)a, y = *(const double *)b;
    return (x > y) - (x < y);
}

long oracle_quantile_rank(long n, double keep)
{
    double r = floor((1.0 - keep) * (double)n);
    long rank = (long)r;
    if (rank < 0) rank = 0;
    if (rank > n - 1) rank = n - 1;
    return rank;
}

float oracle_order_statistic(const double *v, long n, double keep)
{
    double *tmp = (double *)malloc(sizeof(double) * (size_t)n);
    for (long k = 0; k < n; ++k)
        tmp[k] = fabs(v[k]);
    qsort(tmp, (size_t)n, sizeof(double), cmp_double);
    float tau = (float)tmp[oracle_quantile_rank(n, keep)];
    free(tmp);
    return tau;
}

/* ------------------------------------------------------------------------
 * Histogram quantile [blog "Evidence": per layer at most 200,000 activation
 * samples and a 4,096-bin histogram]. The pages fix no more than that; the
 * readings adopted here make every step plain fp32 arithmetic:
 *   samples: every k-th pooled magnitude, k = ceil(n / max_samples), in
 *            pooled order (|v[0]|, |v[k]|, |v[2k]|, ...);
 *   bins:    `bins` equal bins of width w = m / bins over [0, m], m the largest
 *            sample; sample s falls in bin trunc(fp32(s / w)), and m itself
 *            (and anything rounding to bins) in the top bin;
 *   tau:     fp32(b * w), the lower edge of the bin b holding the sample of
 *            rank floor((1 - keep) * n_s) in ascending order (the rank rule of
 *            the exact order statistic), so tau <= that sample < tau + w.
 * v holds fp32 values (the magnitudes are taken here).
 * ---------------------------------------------------------------------- */
float oracle_hist_quantile(const float *v, long n, double keep, long max_samples, int bins)
{
    long k = (n + max_samples - 1) / max_samples;
    if (k < 1)
        k = 1;
    long ns = (n + k - 1) / k;
    float m = 0.0f;
    for (long i = 0; i < ns; ++i) {
        float a = fabsf(v[i * k]);
        if (a > m)
            m = a;
    }
    if (m == 0.0f)
        return 0.0f;
    const float w = m / (float)bins;
    long *hist = (long *)calloc((size_t)bins, sizeof(long));
    for (long i = 0; i < ns; ++i) {
        float q = fabsf(v[i * k]) / w;
        long b = (long)q;                 /* q >= 0: truncation */
        if (b > bins - 1)
            b = bins - 1;
        hist[b] += 1;
    }
    long rank = oracle_quantile_rank(ns, keep);
    long cum = 0;
    int sel = bins - 1;
    for (int b = 0; b < bins; ++b) {
        if (rank < cum + hist[b]) {
            sel = b;
            break;
        }
        cum += hist[b];
    }
    free(hist);
    return (float)sel * w;
}

void oracle_calibrate(int d_model, int d_ff, int n_cal, const uint16_t *x_cal,
                      const uint8_t *q_up, const float *s_up,
                      const uint8_t *q_gate, const float *s_gate,
                      double keep_x, double keep_s, float *tau_x_out,
                      float *tau_s_out, int n_threads, int act,
                      const uint16_t *pw_up, const uint16_t *pw_gate)
{
    long nx = (long)n_cal * d_model;
    double *ax = (double *)malloc(sizeof(double) * (size_t)nx);
    for (long k = 0; k < nx; ++k)
        ax[k] = bf16_value(x_cal[k]);
    float tau_x = oracle_order_statistic(ax, nx, keep_x);
    free(ax);

    long ns = (long)n_cal * d_ff;
    double *sv = (double *)malloc(sizeof(double) * (size_t)ns);
#ifdef _OPENMP
    if (n_threads <= 0)
        n_threads = omp_get_max_threads();
#pragma omp parallel for num_threads(n_threads) schedule(dynamic, 1)
#else
    (void)n_threads;
#endif
    for (int t = 0; t < n_cal; ++t)
        oracle_stage1_token(d_model, d_ff, x_cal + (size_t)t * d_model, tau_x,
                            q_up, s_up, q_gate, s_gate, 0.0f, NULL, NULL, NULL,
                            sv + (size_t)t * d_ff, NULL, act, pw_up, pw_gate);
    *tau_s_out = oracle_order_statistic(sv, ns, keep_s);
    *tau_x_out = tau_x;
    free(sv);
}

/* Histogram calibration [blog "Evidence"]: as oracle_calibrate, with each
 * threshold the histogram quantile above of the pooled fp32 magnitudes (s~
 * rounded to fp32, pooled token by token, channel by channel). */
void oracle_calibrate_hist(int d_model, int d_ff, int n_cal, const uint16_t *x_cal,
                           const uint8_t *q_up, const float *s_up,
                           const uint8_t *q_gate, const float *s_gate,
                           double keep_x, double keep_s, long max_samples, int bins,
                           float *tau_x_out, float *tau_s_out, int n_threads, int act,
                           const uint16_t *pw_up, const uint16_t *pw_gate)
{
    long nx = (long)n_cal * d_model;
    float *ax = (float *)malloc(sizeof(float) * (size_t)nx);
    for (long k = 0; k < nx; ++k)
        ax[k] = bf16_value_f(x_cal[k]);
    float tau_x = oracle_hist_quantile(ax, nx, keep_x, max_samples, bins);
    free(ax);

    long ns = (long)n_cal * d_ff;
    double *sv = (double *)malloc(sizeof(double) * (size_t)ns);
#ifdef _OPENMP
    if (n_threads <= 0)
        n_threads = omp_get_max_threads();
#pragma omp parallel for num_threads(n_threads) schedule(dynamic, 1)
#else
    (void)n_threads;
#endif
    for (int t = 0; t < n_cal; ++t)
        oracle_stage1_token(d_model, d_ff, x_cal + (size_t)t * d_model, tau_x,
                            q_up, s_up, q_gate, s_gate, 0.0f, NULL, NULL, NULL,
                            sv + (size_t)t * d_ff, NULL, act, pw_up, pw_gate);
    float *sf = (float *)malloc(sizeof(float) * (size_t)ns);
    for (long k = 0; k < ns; ++k)
        sf[k] = (float)sv[k];
    *tau_s_out = oracle_hist_quantile(sf, ns, keep_s, max_samples, bins);
    *tau_x_out = tau_x;
    free(sf);
    free(sv);
}

/* ------------------------------------------------------------------------
 * Compute-budget split [blog "Compute budget"]:
 *   C = 2 alpha (1 - s1) + 3 (1 - s2),  e = 1 - C/3 = s2 - 2 alpha (1 - s1)/3.
 * Reading adopted for the allocation rule: anchor s2 at s2_anchor, solve e
 * for s1; if s1 falls outside [0, s1_max], clamp it and solve e for s2.
 * (The blog's worked case: e = 0.7, anchor 0.7, alpha = 1/3 gives s1 = 1,
 * which is clamped to 0.7, so s2 = 0.7 + 2(1/3)(0.3)/3 ~= 0.7667.)
 * ---------------------------------------------------------------------- */
void oracle_allocate(double e, double alpha, double s1_max, double s2_anchor,
                     double *s1_out, double *s2_out)
{
    double s2 = s2_anchor;
    double s1 = 1.0 - 3.0 * (s2 - e) / (2.0 * alpha);
    if (s1 > s1_max || s1 < 0.0) {
        s1 = s1 > s1_max ? s1_max : 0.0;
        s2 = e + 2.0 * alpha * (1.0 - s1) / 3.0;
    }
    *s1_out = s1;
    *s2_out = s2;
}

/* Effective sparsity of a split [blog "Compute budget"]. */
double oracle_effective_sparsity(double s1, double s2, double alpha)
{
    return s2 - 2.0 * alpha * (1.0 - s1) / 3.0;
}

/*
 * Layer stack (the stacked-layer benchmark built on the Prox FFN; not on the
 * Prox pages): pre-norm, h <- h + FFN(RMSNorm(h)), RMSNorm(h) = h /
 * sqrt(mean(h^2) + eps) with unit gain, the FFN input rounded to bf16.
 */

/* nearest bf16 to v, ties to even, as a bit pattern (finite v in range) */
static uint16_t bf16_round(double v)
{
    if (v == 0.0)
        return (uint16_t)(signbit(v) ? 0x8000u : 0u);
    int e;
    frexp(fabs(v), &e);                 /* |v| in [2^(e-1), 2^e) */
    int qexp = e - 8;                   /* 8 significant bits */
    if (qexp < -133)
        qexp = -133;                    /* bf16 subnormal spacing */
    const double q = ldexp(1.0, qexp);
    const double r = nearbyint(fabs(v) / q) * q;    /* default mode: ties to even */
    const float f = (float)(signbit(v) ? -r : r);   /* exact: <= 8 significant bits */
    uint32_t bits;
    memcpy(&bits, &f, sizeof bits);
    return (uint16_t)(bits >> 16);
}

/* one token: x = bf16(h / sqrt(mean(h^2) + eps)), h read exactly */
void oracle_rmsnorm_bf16(int d, const float *h, double eps, uint16_t *x_out)
{
    double ss = 0.0;
    for (int i = 0; i < d; ++i)
        ss += (double)h[i] * (double)h[i];
    const double rms = sqrt(ss / (double)d + eps);
    for (int i = 0; i < d; ++i)
        x_out[i] = bf16_round((double)h[i] / rms);
}

