/*
 * mea_oracle.c -- plain, slow, double-precision CPU oracle for the
 * memory-efficient activation path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product (the CUDA library and its
 * Python binding) links, loads or calls this file.  Only the test-suite, the
 * smoke check and the CPU-baseline leg of the benchmark use it.  It shares no
 * code, header, constant or helper with the CUDA path.
 *
 * Every function takes its inputs as exact doubles (the caller widens the
 * stored bf16 / fp32 values, which is exact) and returns the mathematically
 * defined result evaluated in double with libm.  Comparison against a GPU
 * result happens after rounding the double result to the output storage type
 * (oracle_round_bf16 / oracle_round_f32 below).
 *
 * Sources, by page and section:
 *  - "Memory efficient Swish" (adeeplearner blog, 2021-05-17), sections
 *    "What is a Swish activation function?" and "How is Swish implemented?":
 *    Swish(x) = x * Sigmoid(alpha x), Sigmoid(v) = 1 / (1 + e^-v).
 *  - same page, "How is the memory efficient version Swish implemented?" and
 *    "What makes this implementation save GPU memory?": the forward keeps only
 *    x, the backward recomputes the sigmoid from x and returns
 *    dy * s * (1 + x (1 - s)) at alpha = 1 (product-rule derivation, with
 *    e^-x / (1 + e^-x) rewritten as 1 - Sigmoid(x)).
 *  - "What activations cost, in memory and in arithmetic" (asifuddin.com,
 *    problem B07), GIVEN: the activation family ReLU, LeakyReLU, sigmoid,
 *    tanh, GELU (erf) and GELU (tanh approximation).  The page names them
 *    only; the definitions used here are the standard ones.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - alpha is one scalar per tensor; the derivative in x generalises by the
 *    chain rule to s + alpha x s sigma(-alpha x); d alpha is the derivative of
 *    sum(dy * y) in alpha, i.e. sum(dy * x^2 * s * sigma(-alpha x)).
 *  - 1 - Sigmoid(v) is evaluated as Sigmoid(-v) (the same value, without the
 *    cancellation that 1 - s suffers when s is close to 1).
 *  - ReLU'(0) = 0 and LeakyReLU'(0) = slope (the derivative is the predicate
 *    x > 0).  A NaN input fails that predicate.
 *  - GELU-tanh uses the published constants sqrt(2/pi) and 0.044715
 *    (Hendrycks and Gimpel, 2016); 1 + tanh(u) is evaluated as 2 Sigmoid(2u).
 *  - Fused affine + Swish: z = gamma_c x + beta_c, y = z Sigmoid(z) (alpha 1),
 *    channel c = i mod C for NHWC and (i / (H W)) mod C for NCHW.
 *  - Concatenation + batch normalization + ReLU ("A memory-efficient
 *    implementation of DenseNets", section "Motivation": the outputs of every
 *    concatenation and batch normalization live in shared allocations and
 *    are re-populated in the backward).  The page names the operations only;
 *    batch normalization here is the standard training-mode definition:
 *    per-channel mean and biased variance over N, H, W, xhat = (x - mean) /
 *    sqrt(var + eps), y = max(gamma xhat + beta, 0); running statistics move
 *    by momentum towards the batch mean and the unbiased variance
 *    (oracle_bn_running_update).  The caller concatenates the pieces (along
 *    channels) before calling.
 *  - Matmul + activation (problem B07, SOLUTION step 4: the activation
 *    follows a d x d matrix multiply on the same tensor): Z = X W^T with X
 *    [M x K] and W [N x K] row-major; the activation is evaluated at Z as
 *    stored (rounded to bf16 when the caller asks), because the backward
 *    recomputes it from that stored Z.  The backward of the pair is
 *    dZ = (G W) * f'(Z) for an upstream G [M x K] and W [N x K].
 *
 * Reductions (d alpha, d gamma, d beta) are serial sums in index order in
 * long double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Activation ids of this oracle (its own numbering; the Python wrapper maps
 * activation names onto it). */
enum {
    OR_RELU = 0,
    OR_LEAKY_RELU = 1,
    OR_SIGMOID = 2,
    OR_TANH = 3,
    OR_GELU_ERF = 4,
    OR_GELU_TANH = 5,
    OR_SWISH = 6,
    OR_NUM_ACTS = 7
};

enum { OR_NCHW = 0, OR_NHWC = 1 };

/* ---------------------------------------------------------------- sigmoid */

/* Sigmoid(v) = 1 / (1 + e^-v).  For v < 0 the equal form e^v / (1 + e^v) is
 * used so that e^-v never overflows; both forms are the definition. */
static double sigm(double v)
{
    if (v != v) return v;
    if (v >= 0.0) return 1.0 / (1.0 + exp(-v));
    double e = exp(v);
    return e / (1.0 + e);
}

/* ------------------------------------------------------------------ Swish */

static double swish_f(double x, double alpha)
{
    return x * sigm(alpha * x);
}

/* d/dx [x Sigmoid(alpha x)] = s + alpha x s (1 - s), with (1 - s) taken as
 * Sigmoid(-alpha x). */
static double swish_df(double x, double alpha)
{
    double z = alpha * x;
    double s = sigm(z);
    return s + z * s * sigm(-z);
}

/* d/dalpha [x Sigmoid(alpha x)] = x^2 s (1 - s). */
static double swish_dalpha_term(double x, double alpha)
{
    double z = alpha * x;
    return x * x * sigm(z) * sigm(-z);
}

/* ------------------------------------------------------------ the family */

static double relu_f(double x)
{
    if (x != x) return x;
    return x > 0.0 ? x : 0.0;
}

static double relu_df(double x)
{
    return x > 0.0 ? 1.0 : 0.0;
}

static double leaky_f(double x, double slope)
{
    return x > 0.0 ? x : slope * x;
}

static double leaky_df(double x, double slope)
{
    return x > 0.0 ? 1.0 : slope;
}

static double sigmoid_f(double x)
{
    return sigm(x);
}

/* Sigmoid' = s (1 - s) = Sigmoid(x) Sigmoid(-x). */
static double sigmoid_df(double x)
{
    return sigm(x) * sigm(-x);
}

static double tanh_f(double x)
{
    return tanh(x);
}

/* tanh' = 1 - tanh^2 = 4 Sigmoid(2x) Sigmoid(-2x) (no cancellation). */
static double tanh_df(double x)
{
    return 4.0 * sigm(2.0 * x) * sigm(-2.0 * x);
}

/* Standard normal CDF Phi(x) = erfc(-x / sqrt 2) / 2 and density phi(x). */
static double std_normal_cdf(double x)
{
    return 0.5 * erfc(-x / sqrt(2.0));
}

static double std_normal_pdf(double x)
{
    return exp(-0.5 * x * x) / sqrt(2.0 * M_PI);
}

/* GELU (erf form): x Phi(x). */
static double gelu_erf_f(double x)
{
    return x * std_normal_cdf(x);
}

/* d/dx [x Phi(x)] = Phi(x) + x phi(x). */
static double gelu_erf_df(double x)
{
    return std_normal_cdf(x) + x * std_normal_pdf(x);
}

/* GELU (tanh approximation): x (1 + tanh u) / 2 = x Sigmoid(2u),
 * u = sqrt(2/pi) (x + 0.044715 x^3). */
static const double GELU_K0 = 0.7978845608028654;   /* sqrt(2 / pi) */
static const double GELU_K1 = 0.044715;

static double gelu_tanh_u(double x)
{
    return GELU_K0 * (x + GELU_K1 * x * x * x);
}

static double gelu_tanh_f(double x)
{
    return x * sigm(2.0 * gelu_tanh_u(x));
}

/* d/dx [x Sigmoid(2u)] = Sigmoid(2u) + x 2u' Sigmoid(2u) Sigmoid(-2u),
 * u' = sqrt(2/pi) (1 + 3 * 0.044715 x^2). */
static double gelu_tanh_df(double x)
{
    double v = 2.0 * gelu_tanh_u(x);
    double dv = 2.0 * GELU_K0 * (1.0 + 3.0 * GELU_K1 * x * x);
    double s = sigm(v);
    return s + x * dv * s * sigm(-v);
}

static double act_f(int act, double x, double param)
{
    switch (act) {
    case OR_RELU: return relu_f(x);
    case OR_LEAKY_RELU: return leaky_f(x, param);
    case OR_SIGMOID: return sigmoid_f(x);
    case OR_TANH: return tanh_f(x);
    case OR_GELU_ERF: return gelu_erf_f(x);
    case OR_GELU_TANH: return gelu_tanh_f(x);
    case OR_SWISH: return swish_f(x, param);
    }
    return NAN;
}

static double act_df(int act, double x, double param)
{
    switch (act) {
    case OR_RELU: return relu_df(x);
    case OR_LEAKY_RELU: return leaky_df(x, param);
    case OR_SIGMOID: return sigmoid_df(x);
    case OR_TANH: return tanh_df(x);
    case OR_GELU_ERF: return gelu_erf_df(x);
    case OR_GELU_TANH: return gelu_tanh_df(x);
    case OR_SWISH: return swish_df(x, param);
    }
    return NAN;
}

/* ------------------------------------------------------- exported: family */

/* y[i] = f(x[i]; param).  param is alpha for Swish, the slope for
 * LeakyReLU, ignored otherwise.  Returns 0, or -1 for an unknown act. */
int oracle_act_fwd(int act, const double *x, double *y, int64_t n, double param)
{
    if (act < 0 || act >= OR_NUM_ACTS || n < 0) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) y[i] = act_f(act, x[i], param);
    return 0;
}

/* dx[i] = dy[i] * f'(x[i]; param), with f' recomputed from x alone. */
int oracle_act_bwd(int act, const double *x, const double *dy, double *dx,
                   int64_t n, double param)
{
    if (act < 0 || act >= OR_NUM_ACTS || n < 0) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) dx[i] = dy[i] * act_df(act, x[i], param);
    return 0;
}

/* The derivative alone (dy = 1), for closed-form and finite-difference
 * checks. */
int oracle_act_deriv(int act, const double *x, double *d, int64_t n, double param)
{
    if (act < 0 || act >= OR_NUM_ACTS || n < 0) return -1;
    for (int64_t i = 0; i < n; ++i) d[i] = act_df(act, x[i], param);
    return 0;
}

/* Condition scale of the backward product dx = dy f'(x): |dy| times the sum
 * of the absolute values of the terms f' is made of.  Where f' is a sum
 * whose terms cancel (Swish and both GELUs near the zero of f'), the error
 * of any finite-precision evaluation is proportional to this scale rather
 * than to |dx|; elsewhere it equals |dx|.  Used by the tests to state the
 * fp32 tolerance as |g - r| <= 1e-5 max(|r|, scale). */
static double act_df_abs_terms(int act, double x, double param)
{
    switch (act) {
    case OR_SWISH: {
        double z = param * x, s = sigm(z);
        return s + fabs(z) * s * sigm(-z);
    }
    case OR_GELU_ERF:
        return std_normal_cdf(x) + fabs(x) * std_normal_pdf(x);
    case OR_GELU_TANH: {
        double v = 2.0 * gelu_tanh_u(x);
        double dv = 2.0 * GELU_K0 * (1.0 + 3.0 * GELU_K1 * x * x);
        double s = sigm(v);
        return s + fabs(x * dv) * s * sigm(-v);
    }
    default:
        return fabs(act_df(act, x, param));
    }
}

int oracle_act_bwd_scale(int act, const double *x, const double *dy, double *m,
                         int64_t n, double param)
{
    if (act < 0 || act >= OR_NUM_ACTS || n < 0) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) m[i] = fabs(dy[i]) * act_df_abs_terms(act, x[i], param);
    return 0;
}

/* d alpha = sum_i dy_i x_i^2 s_i (1 - s_i), serial, index order, long
 * double accumulator. */
double oracle_swish_dalpha(const double *x, const double *dy, int64_t n, double alpha)
{
    long double acc = 0.0L;
    for (int64_t i = 0; i < n; ++i)
        acc += (long double)(dy[i] * swish_dalpha_term(x[i], alpha));
    return (double)acc;
}

/* ------------------------------------------------ exported: affine + Swish */

static int64_t channel_of(int layout, const int64_t shape[4], int64_t i)
{
    int64_t C = shape[1], HW = shape[2] * shape[3];
    if (layout == OR_NHWC) return i % C;
    return (i / HW) % C;
}

/* y = z Sigmoid(z), z = gamma_c x + beta_c; shape = {N, C, H, W} in both
 * layouts (the layout says how the flat index maps to a channel). */
int oracle_affine_swish_fwd(int layout, const int64_t shape[4], const double *x,
                            const double *gamma, const double *beta, double *y)
{
    if (layout != OR_NCHW && layout != OR_NHWC) return -1;
    int64_t n = shape[0] * shape[1] * shape[2] * shape[3];
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        int64_t c = channel_of(layout, shape, i);
        double z = gamma[c] * x[i] + beta[c];
        y[i] = z * sigm(z);
    }
    return 0;
}

/* dz = dy (s + z s (1 - s)); dx = gamma_c dz; dgamma_c = sum dz x;
 * dbeta_c = sum dz (serial, index order, long double).  dx_scale, when not
 * NULL, receives the condition scale of each dx (see oracle_act_bwd_scale). */
int oracle_affine_swish_bwd(int layout, const int64_t shape[4], const double *x,
                            const double *dy, const double *gamma, const double *beta,
                            double *dx, double *dgamma, double *dbeta, double *dx_scale)
{
    if (layout != OR_NCHW && layout != OR_NHWC) return -1;
    int64_t C = shape[1];
    int64_t n = shape[0] * shape[1] * shape[2] * shape[3];
    long double *acc_g = (long double *)calloc((size_t)(C > 0 ? C : 1), sizeof(long double));
    long double *acc_b = (long double *)calloc((size_t)(C > 0 ? C : 1), sizeof(long double));
    if (!acc_g || !acc_b) { free(acc_g); free(acc_b); return -2; }
    for (int64_t i = 0; i < n; ++i) {
        int64_t c = channel_of(layout, shape, i);
        double z = gamma[c] * x[i] + beta[c];
        double s = sigm(z);
        double dz = dy[i] * (s + z * s * sigm(-z));
        dx[i] = gamma[c] * dz;
        if (dx_scale)   /* condition scale of dx (see oracle_act_bwd_scale) */
            dx_scale[i] = fabs(gamma[c] * dy[i]) * (s + fabs(z) * s * sigm(-z));
        acc_g[c] += (long double)(dz * x[i]);
        acc_b[c] += (long double)dz;
    }
    for (int64_t c = 0; c < C; ++c) {
        dgamma[c] = (double)acc_g[c];
        dbeta[c] = (double)acc_b[c];
    }
    free(acc_g);
    free(acc_b);
    return 0;
}

/* ------------------------------------ exported: per-channel family (NEXT) */

/* Per-channel affine followed by any activation of the family:
 * z = gamma_c x + beta_c, y = f(z; param).  The affine + Swish functions above
 * are the case act = Swish, param = 1. */
int oracle_affine_act_fwd(int act, int layout, const int64_t shape[4], const double *x,
                          const double *gamma, const double *beta, double param, double *y)
{
    if (act < 0 || act >= OR_NUM_ACTS || (layout != OR_NCHW && layout != OR_NHWC)) return -1;
    int64_t n = shape[0] * shape[1] * shape[2] * shape[3];
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        int64_t c = channel_of(layout, shape, i);
        y[i] = act_f(act, gamma[c] * x[i] + beta[c], param);
    }
    return 0;
}

/* dz = dy f'(z); dx = gamma_c dz; dgamma_c = sum dz x; dbeta_c = sum dz
 * (serial, index order, long double).  dx_scale (nullable) receives
 * |gamma_c| times the condition scale of dy f'(z) (see oracle_act_bwd_scale). */
int oracle_affine_act_bwd(int act, int layout, const int64_t shape[4], const double *x,
                          const double *dy, const double *gamma, const double *beta, double param,
                          double *dx, double *dgamma, double *dbeta, double *dx_scale)
{
    if (act < 0 || act >= OR_NUM_ACTS || (layout != OR_NCHW && layout != OR_NHWC)) return -1;
    int64_t C = shape[1];
    int64_t n = shape[0] * shape[1] * shape[2] * shape[3];
    long double *acc_g = (long double *)calloc((size_t)(C > 0 ? C : 1), sizeof(long double));
    long double *acc_b = (long double *)calloc((size_t)(C > 0 ? C : 1), sizeof(long double));
    if (!acc_g || !acc_b) { free(acc_g); free(acc_b); return -2; }
    for (int64_t i = 0; i < n; ++i) {
        int64_t c = channel_of(layout, shape, i);
        double z = gamma[c] * x[i] + beta[c];
        double dz = dy[i] * act_df(act, z, param);
        dx[i] = gamma[c] * dz;
        if (dx_scale) dx_scale[i] = fabs(gamma[c] * dy[i]) * act_df_abs_terms(act, z, param);
        acc_g[c] += (long double)(dz * x[i]);
        acc_b[c] += (long double)dz;
    }
    for (int64_t c = 0; c < C; ++c) {
        dgamma[c] = (double)acc_g[c];
        dbeta[c] = (double)acc_b[c];
    }
    free(acc_g);
    free(acc_b);
    return 0;
}

/* How much the affine outputs move when z = gamma_c x + beta_c is rounded
 * once to binary32.  Any fp32 evaluation (the configurations compute in fp32)
 * forms z in binary32, which moves it by at most u |z|, u = 2^-24 (round to
 * nearest); no arithmetic after that rounding can recover the exact z.  For
 * each element: ey = the largest change of y = f(z), and edx = the largest
 * change of dx = gamma_c dy f'(z), when z moves to z (1 - u) or z (1 + u),
 * evaluated in double as differences of the definitions at those points.
 * Near-linear f gives ey = u |z f'(z)| and edx = u |z gamma_c dy f''(z)| to
 * first order.  The tests add these to the fp32 tolerance of the affine
 * outputs. */
int oracle_affine_act_zround(int act, int layout, const int64_t shape[4], const double *x, const double *dy,
                             const double *gamma, const double *beta, double param, double *ey, double *edx)
{
    if (act < 0 || act >= OR_NUM_ACTS || (layout != OR_NCHW && layout != OR_NHWC)) return -1;
    const double u = ldexp(1.0, -24);
    int64_t n = shape[0] * shape[1] * shape[2] * shape[3];
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        int64_t c = channel_of(layout, shape, i);
        double z = gamma[c] * x[i] + beta[c];
        double lo = z * (1.0 - u), hi = z * (1.0 + u);
        double f0 = act_f(act, z, param), d0 = act_df(act, z, param);
        double fy = fmax(fabs(act_f(act, lo, param) - f0), fabs(act_f(act, hi, param) - f0));
        double fd = fmax(fabs(act_df(act, lo, param) - d0), fabs(act_df(act, hi, param) - d0));
        ey[i] = fy;
        edx[i] = fabs(gamma[c] * dy[i]) * fd;
    }
    return 0;
}

/* Swish with one alpha per channel: y = x Sigmoid(alpha_c x). */
int oracle_swish_channel_fwd(int layout, const int64_t shape[4], const double *x,
                             const double *alpha, double *y)
{
    if (layout != OR_NCHW && layout != OR_NHWC) return -1;
    int64_t n = shape[0] * shape[1] * shape[2] * shape[3];
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) y[i] = swish_f(x[i], alpha[channel_of(layout, shape, i)]);
    return 0;
}

/* dx = dy Swish'(x; alpha_c); dalpha_c = sum over channel c of
 * dy x^2 s (1 - s) (serial, index order, long double).  dx_scale as above. */
int oracle_swish_channel_bwd(int layout, const int64_t shape[4], const double *x, const double *dy,
                             const double *alpha, double *dx, double *dalpha, double *dx_scale)
{
    if (layout != OR_NCHW && layout != OR_NHWC) return -1;
    int64_t C = shape[1];
    int64_t n = shape[0] * shape[1] * shape[2] * shape[3];
    long double *acc = (long double *)calloc((size_t)(C > 0 ? C : 1), sizeof(long double));
    if (!acc) return -2;
    for (int64_t i = 0; i < n; ++i) {
        int64_t c = channel_of(layout, shape, i);
        dx[i] = dy[i] * swish_df(x[i], alpha[c]);
        if (dx_scale) dx_scale[i] = fabs(dy[i]) * act_df_abs_terms(OR_SWISH, x[i], alpha[c]);
        acc[c] += (long double)(dy[i] * swish_dalpha_term(x[i], alpha[c]));
    }
    for (int64_t c = 0; c < C; ++c) dalpha[c] = (double)acc[c];
    free(acc);
    return 0;
}

/* ------------------------------------------------- matmul + activation */

static uint16_t bf16_from_double(double v);

static double bf16_value(double v)
{
    union {
        uint32_t u;
        float f;
    } b;
    b.u = (uint32_t)bf16_from_double(v) << 16;
    return (double)b.f;
}

/* Z[m][n] = sum_k X[m][k] W[n][k]  (serial over k, long double);
 * Y[m][n] = f(z) with z = Z[m][n], or z = Z[m][n] rounded to the nearest
 * bf16 when round_z_bf16 is non-zero (the value a bf16 store of Z holds).
 * absum (nullable) receives sum_k |X[m][k] W[n][k]|, the scale of the
 * rounding error of any floating-point evaluation of the sum.  Y may be NULL. */
int oracle_matmul_act_fwd(int act, int64_t M, int64_t N, int64_t K, const double *X, const double *W,
                          double param, int round_z_bf16, double *Z, double *Y, double *absum)
{
    if (act < 0 || act >= OR_NUM_ACTS || M < 0 || N < 0 || K < 0) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            long double acc = 0.0L, aacc = 0.0L;
            for (int64_t k = 0; k < K; ++k) {
                long double t = (long double)X[m * K + k] * (long double)W[n * K + k];
                acc += t;
                aacc += fabsl(t);
            }
            double z = (double)acc;
            Z[m * N + n] = z;
            if (absum) absum[m * N + n] = (double)aacc;
            if (Y) Y[m * N + n] = act_f(act, round_z_bf16 ? bf16_value(z) : z, param);
        }
    }
    return 0;
}

/* D[m][n] = sum_k G[m][k] W[n][k] (serial over k, long double) and
 * dZ[m][n] = D[m][n] f'(Z[m][n]), Z as stored.  D and absum (sum_k
 * |G[m][k] W[n][k]|) are nullable. */
int oracle_matmul_act_bwd(int act, int64_t M, int64_t N, int64_t K, const double *G, const double *W,
                          const double *Z, double param, double *dZ, double *D, double *absum)
{
    if (act < 0 || act >= OR_NUM_ACTS || M < 0 || N < 0 || K < 0) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            long double acc = 0.0L, aacc = 0.0L;
            for (int64_t k = 0; k < K; ++k) {
                long double t = (long double)G[m * K + k] * (long double)W[n * K + k];
                acc += t;
                aacc += fabsl(t);
            }
            double d = (double)acc;
            if (D) D[m * N + n] = d;
            if (absum) absum[m * N + n] = (double)aacc;
            dZ[m * N + n] = d * act_df(act, Z[m * N + n], param);
        }
    }
    return 0;
}

/* ---------------------------------------- batch normalization + ReLU */

/* x: NCHW [N, C, HW] (channel c of sample n is the plane x[(n C + c) HW ..]).
 * Outputs: y = max(gamma xhat + beta, 0); mean[c], var[c] (biased); y_scale
 * (nullable) = |gamma| r |x| + |gamma| r |mean| + |beta|, r = 1 / sqrt(var +
 * eps): the magnitude of the terms any evaluation of gamma xhat + beta adds.
 * Sums are serial in index order, long double, two passes (mean first). */
int oracle_bn_relu_fwd(int64_t N, int64_t C, int64_t HW, const double *x, const double *gamma,
                       const double *beta, double eps, double *y, double *mean, double *var, double *y_scale)
{
    if (N < 0 || C < 0 || HW < 0) return -1;
    const int64_t n = N * HW;
#pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < C; ++c) {
        long double s = 0.0L;
        for (int64_t b = 0; b < N; ++b)
            for (int64_t i = 0; i < HW; ++i) s += (long double)x[(b * C + c) * HW + i];
        const long double mu = n > 0 ? s / (long double)n : 0.0L;
        long double v = 0.0L;
        for (int64_t b = 0; b < N; ++b)
            for (int64_t i = 0; i < HW; ++i) {
                const long double d = (long double)x[(b * C + c) * HW + i] - mu;
                v += d * d;
            }
        const long double var_c = n > 0 ? v / (long double)n : 0.0L;
        mean[c] = (double)mu;
        var[c] = (double)var_c;
        const double r = 1.0 / sqrt((double)var_c + eps);
        for (int64_t b = 0; b < N; ++b)
            for (int64_t i = 0; i < HW; ++i) {
                const int64_t j = (b * C + c) * HW + i;
                const double xh = (x[j] - (double)mu) * r;
                const double z = gamma[c] * xh + beta[c];
                y[j] = z > 0.0 ? z : 0.0;
                if (y_scale) y_scale[j] = fabs(gamma[c]) * r * (fabs(x[j]) + fabs((double)mu)) + fabs(beta[c]);
            }
    }
    return 0;
}

/* Backward of y = max(gamma xhat + beta, 0) with batch statistics, from x,
 * dy and the batch mean / biased variance (nothing else saved):
 *   dz = dy [gamma xhat + beta > 0];  dbeta = sum dz;  dgamma = sum dz xhat;
 *   dx = gamma r (dz - dbeta / n - xhat dgamma / n).
 * dx_scale (nullable) = |gamma| r (|dz| + sum|dz| / n + |xhat| sum|dz xhat| / n),
 * the magnitude of the terms that dx adds up. */
int oracle_bn_relu_bwd(int64_t N, int64_t C, int64_t HW, const double *x, const double *dy, const double *gamma,
                       const double *beta, const double *mean, const double *var, double eps, double *dx,
                       double *dgamma, double *dbeta, double *dx_scale)
{
    if (N < 0 || C < 0 || HW < 0) return -1;
    const int64_t n = N * HW;
#pragma omp parallel for schedule(static)
    for (int64_t c = 0; c < C; ++c) {
        const double r = 1.0 / sqrt(var[c] + eps);
        long double sdz = 0.0L, sdzx = 0.0L, adz = 0.0L, adzx = 0.0L;
        for (int64_t b = 0; b < N; ++b)
            for (int64_t i = 0; i < HW; ++i) {
                const int64_t j = (b * C + c) * HW + i;
                const double xh = (x[j] - mean[c]) * r;
                const double dz = gamma[c] * xh + beta[c] > 0.0 ? dy[j] : 0.0;
                sdz += (long double)dz;
                sdzx += (long double)dz * (long double)xh;
                adz += fabsl((long double)dz);
                adzx += fabsl((long double)dz * (long double)xh);
            }
        dbeta[c] = (double)sdz;
        dgamma[c] = (double)sdzx;
        const double k = gamma[c] * r;
        for (int64_t b = 0; b < N; ++b)
            for (int64_t i = 0; i < HW; ++i) {
                const int64_t j = (b * C + c) * HW + i;
                const double xh = (x[j] - mean[c]) * r;
                const double dz = gamma[c] * xh + beta[c] > 0.0 ? dy[j] : 0.0;
                dx[j] = n > 0 ? k * (dz - (double)sdz / (double)n - xh * (double)sdzx / (double)n) : 0.0;
                if (dx_scale)
                    dx_scale[j] = n > 0 ? fabs(k) * (fabs(dz) + (double)adz / (double)n +
                                                     fabs(xh) * (double)adzx / (double)n)
                                        : 0.0;
            }
    }
    return 0;
}

/* Running statistics after one training step of batch normalization, per
 * channel: running_mean <- (1 - momentum) running_mean + momentum mean and
 * running_var <- (1 - momentum) running_var + momentum var n / (n - 1), the
 * unbiased batch variance over n = N H W values (standard training-mode
 * definition).  For n = 1 the unbiased variance is undefined; the biased one
 * (zero) is used.  running_mean and running_var are updated in place. */
int oracle_bn_running_update(int64_t C, int64_t n, const double *mean, const double *var, double momentum,
                             double *running_mean, double *running_var)
{
    if (C < 0 || n < 1) return -1;
    for (int64_t c = 0; c < C; ++c) {
        double unbiased = n > 1 ? var[c] * (double)n / (double)(n - 1) : var[c];
        running_mean[c] = (1.0 - momentum) * running_mean[c] + momentum * mean[c];
        running_var[c] = (1.0 - momentum) * running_var[c] + momentum * unbiased;
    }
    return 0;
}

/* ------------------------------------------------------ storage rounding */

/* Round a double to the nearest bfloat16 (1 sign bit, 8 exponent bits with
 * bias 127, 7 stored mantissa bits), ties to even, and return its bit
 * pattern.  Written from the format's definition: find the spacing of
 * representable values around |v| (2^(e-7) in the binade [2^e, 2^(e+1)),
 * 2^-133 in the subnormal range), round |v| / spacing to an integer with
 * ties to even, and encode.  Values at or beyond the rounding boundary above
 * the largest finite bf16 become infinity. */
static uint16_t bf16_from_double(double v)
{
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    if (v != v) return (uint16_t)(sign | 0x7fc0u);
    double a = fabs(v);
    if (a == 0.0) return sign;
    if (isinf(a)) return (uint16_t)(sign | 0x7f80u);
    int e2;
    frexp(a, &e2);          /* a in [2^(e2-1), 2^e2) */
    int e = e2 - 1;
    if (e < -126) e = -126; /* subnormals share the spacing of the lowest binade */
    double spacing = ldexp(1.0, e - 7);
    double q = nearbyint(a / spacing);   /* default rounding: ties to even */
    double r = q * spacing;
    double max_finite = ldexp(255.0, 120); /* (2 - 2^-7) * 2^127 */
    if (r > max_finite) return (uint16_t)(sign | 0x7f80u);
    if (r == 0.0) return sign;
    int re2;
    frexp(r, &re2);
    int re = re2 - 1;
    if (re < -126) {
        /* subnormal: value = m * 2^-133, m in 1..127 */
        uint16_t m = (uint16_t)ldexp(r, 133);
        return (uint16_t)(sign | m);
    }
    uint16_t m = (uint16_t)(ldexp(r, 7 - re) - 128.0); /* stored mantissa 0..127 */
    uint16_t ex = (uint16_t)(re + 127);
    return (uint16_t)(sign | (ex << 7) | m);
}

void oracle_round_bf16(const double *v, uint16_t *out, int64_t n)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = bf16_from_double(v[i]);
}

/* Round to binary32 with ties to even (C's conversion in the default
 * rounding mode). */
void oracle_round_f32(const double *v, float *out, int64_t n)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = (float)v[i];
}

/* Threads the OpenMP loops use from now on (the baseline's single-core
 * figure); n < 1 is ignored. */
void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n >= 1) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
