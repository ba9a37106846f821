/*
 * CPU ORACLE for the gpt-oss MoE feed-forward block -- TEST INFRASTRUCTURE.
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference
 * leg may load or call this library.  The CUDA product path never does; the
 * two share no code.
 *
 * Plain loops in fp64, one token after another, in the order the block is
 * described:
 *   1. RMSNorm: xn = x / RMS(x) * scale, with RMS(x) = sqrt(mean(x^2) + eps)
 *      ("gpt-oss-20B" hub page, section 3.2 "RMSNorm"; the pnsm.cn overview,
 *      section 2.3 says it has no bias and no mean subtraction).  The pages
 *      give no eps; the caller passes it (1e-5 in every workload).
 *   2. Linear router with bias on xn: logit_e = W_r[e,:] . xn + b_e
 *      ("gpt-oss-20B" page, section 3.4 "混合专家").  The logits are rounded
 *      to fp32 -- the routing decision is taken on fp32 logits.
 *   3. Top-k (k = 4) of the logits, ties to the lower expert index
 *      (pnsm.cn overview section 2.2; config.json read-out on youleyou.com:
 *      experts_per_token 4).
 *   4. Softmax over the k chosen logits (pnsm.cn overview section 2.2: the
 *      chosen experts' outputs are weighted by a softmax over them;
 *      "gpt-oss-20B" page section 3.4).
 *   5. Per chosen expert, gated SwiGLU with the clamp at 7 and the "+1"
 *      ("gpt-oss-20B" page section 3.3 "SwiGLU：带有夹断和残差的门控激活"):
 *        z = W13 xn + b13 (2F values: rows [0,F) gate, [F,2F) linear)
 *        g = min(z_gate, 7);  u = clamp(z_lin, -7, 7)
 *        h = g * sigmoid(1.702 g) * (u + 1)
 *        o = W2 h + b2
 *      with W13 and W2 stored as MXFP4 (pnsm.cn overview sections 1 and 4:
 *      MoE weights in MXFP4 at about 4.25 bits per weight): E2M1 codes
 *      {0, .5, 1, 1.5, 2, 3, 4, 6} with a sign bit, 32 consecutive elements of a
 *      row (along the reduction axis) share one E8M0 scale 2^(s-127);
 *      element 2m of a row is the low nibble of byte m.
 *   6. y = x + sum_i w_i * o_i  (weighted combine and the block residual).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- formats */

static double bf16_value(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Magnitudes of the eight non-negative E2M1 codes, indexed by the code's low
 * three bits (two exponent bits, one mantissa bit); bit 3 is the sign. */
static const double E2M1_MAGNITUDE[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

/* Value of one E2M1 code under an E8M0 scale byte; 255 is NaN. */
double oracle_mxfp4_value(int code, int scale) {
    if (scale == 255) return NAN;
    double v = ldexp(E2M1_MAGNITUDE[code & 7], scale - 127);
    return (code & 8) ? -v : v;
}

/* Storage bytes of an R x K MXFP4 matrix: K/2 code bytes and K/32 scale
 * bytes per row. */
long long oracle_mxfp4_bytes(long long R, long long K) {
    return R * (K / 2) + R * (K / 32);
}

/* Element (r, j) of an R x K MXFP4 matrix. */
static double mx_elem(const uint8_t *codes, const uint8_t *scales, int K, int r, int j) {
    uint8_t byte = codes[(size_t)r * (size_t)(K / 2) + (size_t)(j / 2)];
    int code = (j & 1) ? (byte >> 4) : (byte & 15);
    return oracle_mxfp4_value(code, scales[(size_t)r * (size_t)(K / 32) + (size_t)(j / 32)]);
}

/* Dense decode of an R x K MXFP4 matrix into out[R*K]. */
void oracle_mxfp4_decode_matrix(int R, int K, const uint8_t *codes, const uint8_t *scales, double *out) {
    for (int r = 0; r < R; ++r)
        for (int j = 0; j < K; ++j)
            out[(size_t)r * K + j] = mx_elem(codes, scales, K, r, j);
}

/* Row r of an MXFP4 matrix times a dense vector v[K], in fp64. */
static double mx_row_dot(const uint8_t *codes, const uint8_t *scales, int K, int r, const double *v) {
    double acc = 0.0;
    for (int j = 0; j < K; ++j) acc += mx_elem(codes, scales, K, r, j) * v[j];
    return acc;
}

/* ------------------------------------------------------------ block steps */

/* Step 1: RMSNorm of T rows of length d. */
void oracle_rmsnorm(int T, int d, double eps, const uint16_t *x, const uint16_t *scale, double *xn) {
    for (int t = 0; t < T; ++t) {
        const uint16_t *xt = x + (size_t)t * d;
        double ss = 0.0;
        for (int j = 0; j < d; ++j) {
            double v = bf16_value(xt[j]);
            ss += v * v;
        }
        double inv_rms = 1.0 / sqrt(ss / d + eps);
        for (int j = 0; j < d; ++j) xn[(size_t)t * d + j] = bf16_value(xt[j]) * inv_rms * bf16_value(scale[j]);
    }
}

/* Step 2: router logits of one normalised token, rounded to fp32. */
static void router_token(int d, int E, const double *xn_t, const uint16_t *W, const float *b, float *logit) {
    for (int e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int j = 0; j < d; ++j) acc += bf16_value(W[(size_t)e * d + j]) * xn_t[j];
        logit[e] = (float)(acc + (double)b[e]);
    }
}

void oracle_router(int T, int d, int E, const double *xn, const uint16_t *W, const float *b, float *logits) {
    for (int t = 0; t < T; ++t) router_token(d, E, xn + (size_t)t * d, W, b, logits + (size_t)t * E);
}

/* Steps 3 and 4 for one token: the k largest logits (ties to the lower
 * index), then the softmax over the chosen ones. */
static void topk_softmax_token(int E, int k, const float *logit, int *idx, double *w) {
    for (int i = 0; i < k; ++i) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            int taken = 0;
            for (int p = 0; p < i; ++p) taken |= (idx[p] == e);
            if (taken) continue;
            if (best < 0 || logit[e] > logit[best]) best = e;  /* strict: equal keeps the lower index */
        }
        idx[i] = best;
    }
    double lmax = (double)logit[idx[0]];
    for (int i = 1; i < k; ++i)
        if ((double)logit[idx[i]] > lmax) lmax = (double)logit[idx[i]];
    double sum = 0.0;
    for (int i = 0; i < k; ++i) {
        w[i] = exp((double)logit[idx[i]] - lmax);
        sum += w[i];
    }
    for (int i = 0; i < k; ++i) w[i] /= sum;
}

void oracle_topk_softmax(int T, int E, int k, const float *logits, int *idx, double *w) {
    for (int t = 0; t < T; ++t)
        topk_softmax_token(E, k, logits + (size_t)t * E, idx + (size_t)t * k, w + (size_t)t * k);
}

/* Step 5's activation: gate clamped above at 7, linear part clamped to
 * [-7, 7], alpha = 1.702, and the "+1" on the linear part. */
double oracle_swiglu(double gate, double lin) {
    double g = fmin(gate, 7.0);
    double u = fmax(fmin(lin, 7.0), -7.0);
    return g * (1.0 / (1.0 + exp(-1.702 * g))) * (u + 1.0);
}

/* Step 5 for one token and one expert: o[d] = W2 swiglu(W13 xn + b13) + b2.
 * The weight pointers are the expert's own slices. */
void oracle_expert(int d, int F, const double *xn_t,
                   const uint8_t *w13_codes, const uint8_t *w13_scales, const uint16_t *b13,
                   const uint8_t *w2_codes, const uint8_t *w2_scales, const uint16_t *b2,
                   double *h_out, double *o) {
    double *h = h_out ? h_out : (double *)malloc(sizeof(double) * (size_t)F);
    for (int j = 0; j < F; ++j) {
        double gate = mx_row_dot(w13_codes, w13_scales, d, j, xn_t) + bf16_value(b13[j]);
        double lin = mx_row_dot(w13_codes, w13_scales, d, F + j, xn_t) + bf16_value(b13[F + j]);
        h[j] = oracle_swiglu(gate, lin);
    }
    for (int r = 0; r < d; ++r) o[r] = mx_row_dot(w2_codes, w2_scales, F, r, h) + bf16_value(b2[r]);
    if (!h_out) free(h);
}

/* The whole block for T tokens.  Outputs: y[T*d] (fp64), the chosen experts
 * idx[T*k], their weights w[T*k] and the fp32 router logits[T*E] (each of the
 * last three may be NULL).  Tokens are independent; nthreads > 0 spreads them
 * over that many OpenMP threads (0: the OpenMP default). */
int oracle_moe_forward(int T, int d, int F, int E, int k, double eps,
                       const uint16_t *x, const uint16_t *norm_scale,
                       const uint16_t *router_w, const float *router_b,
                       const uint8_t *w13_codes, const uint8_t *w13_scales, const uint16_t *b13,
                       const uint8_t *w2_codes, const uint8_t *w2_scales, const uint16_t *b2,
                       double *y, int *idx_out, double *w_out, float *logits_out, int nthreads) {
    if (T < 0 || d <= 0 || F <= 0 || E <= 0 || k < 1 || k > E || d % 32 || F % 32) return -1;
    const size_t w13_row_codes = (size_t)d / 2, w13_row_scales = (size_t)d / 32;
    const size_t w2_row_codes = (size_t)F / 2, w2_row_scales = (size_t)F / 32;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int t = 0; t < T; ++t) {
        double *xn = (double *)malloc(sizeof(double) * (size_t)d);
        float *logit = (float *)malloc(sizeof(float) * (size_t)E);
        int *idx = (int *)malloc(sizeof(int) * (size_t)k);
        double *w = (double *)malloc(sizeof(double) * (size_t)k);
        double *o = (double *)malloc(sizeof(double) * (size_t)d);

        oracle_rmsnorm(1, d, eps, x + (size_t)t * d, norm_scale, xn);
        router_token(d, E, xn, router_w, router_b, logit);
        topk_softmax_token(E, k, logit, idx, w);

        double *yt = y + (size_t)t * d;
        for (int j = 0; j < d; ++j) yt[j] = bf16_value(x[(size_t)t * d + j]);
        for (int i = 0; i < k; ++i) {
            size_t e = (size_t)idx[i];
            oracle_expert(d, F, xn,
                          w13_codes + e * 2 * F * w13_row_codes, w13_scales + e * 2 * F * w13_row_scales,
                          b13 + e * 2 * F,
                          w2_codes + e * d * w2_row_codes, w2_scales + e * d * w2_row_scales,
                          b2 + e * d, NULL, o);
            for (int j = 0; j < d; ++j) yt[j] += w[i] * o[j];
        }
        if (idx_out) memcpy(idx_out + (size_t)t * k, idx, sizeof(int) * (size_t)k);
        if (w_out) memcpy(w_out + (size_t)t * k, w, sizeof(double) * (size_t)k);
        if (logits_out) memcpy(logits_out + (size_t)t * E, logit, sizeof(float) * (size_t)E);
        free(xn); free(logit); free(idx); free(w); free(o);
    }
    return 0;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
