/*
 * qknorm_oracle.c -- plain float64 CPU oracle for layerwise Query-Key RMSNorm.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load this library. The product (the CUDA
 * library and its Python binding) never links, loads or calls it, and this
 * file shares no code with it.
 *
 * Source: the SwiftQK technical review ("SwiftQK: When Normalization Becomes
 * the Bottleneck of Tensor Parallelism"):
 *   - "Prerequisites", Eq. (1): RMSNorm(x) = x / sqrt(mean_j x_j^2 + eps) * gamma,
 *     with the mean over the full hidden width H and eps inside the root.
 *   - "Prerequisites", layerwise QK-Norm: one factor per token over the whole
 *     projected Q vector, and separately over the whole projected K vector.
 *   - Section 3, Algorithm 1: Phase A forms the sum of squares of each shard
 *     of the hidden dimension; Phase B adds the shards' scalars and forms
 *     1 / sqrt(S_global / H_total + eps), while x * gamma is formed on its
 *     own; Phase C multiplies the weighted row by that factor.
 *   - Section 4b, Eqs. (3)-(8): the same steps on a worked example.
 *
 * What is computed, in double precision, for one tensor X of width D split
 * into P equal shards of width w = D / P:
 *   S[t,p] = sum_{j = p*w}^{p*w + w - 1} x[t,j]^2      (left to right)
 *   S[t]   = sum_{p = 0}^{P-1} S[t,p]                  (in order of p)
 *   r[t]   = 1 / sqrt(S[t] / D + eps)
 *   y[t,j] = (x[t,j] * gamma[j]) * r[t]                (kept unrounded)
 * x is the stored input (fp32, bf16 given as its 16-bit pattern, or FP8 E4M3
 * given as its 8-bit code), widened
 * exactly to double; gamma is fp32 widened exactly; eps is passed as the
 * double value the caller wants (the fp32 value the GPU receives, widened).
 *
 * Return value of every function: 0 on success, -1 on bad arguments.
 * Rows are independent, so the token loop may run on several threads
 * (nthreads <= 0 means one); the arithmetic of a row does not depend on it.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define QKO_F32 0
#define QKO_BF16 1
#define QKO_E4M3 2

/* Exact value of an FP8 E4M3 code (1 sign, 4 exponent bits with bias 7,
 * 3 mantissa bits; no infinities; S.1111.111 is NaN). */
static double qko_e4m3(uint8_t b)
{
    int sign = b >> 7, e = (b >> 3) & 15, m = b & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);           /* subnormal: m/8 * 2^(1-7) */
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -v : v;
}

/* Exact widening of element i of a stored row to double. */
static double qko_load(const void *x, int dtype, int64_t i)
{
    if (dtype == QKO_F32)
        return (double)((const float *)x)[i];
    if (dtype == QKO_E4M3)
        return qko_e4m3(((const uint8_t *)x)[i]);
    uint32_t bits = (uint32_t)((const uint16_t *)x)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static int qko_check(const void *x, int dtype, int64_t T, int64_t D, int64_t P)
{
    if (T < 0 || D <= 0 || P <= 0 || D % P != 0)
        return -1;
    if (dtype != QKO_F32 && dtype != QKO_BF16 && dtype != QKO_E4M3)
        return -1;
    if (T > 0 && x == NULL)
        return -1;
    return 0;
}

static size_t qko_elem_size(int dtype)
{
    return dtype == QKO_F32 ? 4 : (dtype == QKO_BF16 ? 2 : 1);
}

/* Phase A: per-shard sums of squares of one row, S_row[p] for p < P. */
static void qko_row_partials(const void *row, int dtype, int64_t D, int64_t P, double *S_row)
{
    int64_t w = D / P;
    for (int64_t p = 0; p < P; ++p) {
        double s = 0.0;
        for (int64_t j = p * w; j < p * w + w; ++j) {
            double v = qko_load(row, dtype, j);
            s += v * v;
        }
        S_row[p] = s;
    }
}

/* S[t*P + p] = sum of squares of shard p of row t. */
int qko_partial_sumsq(const void *x, int dtype, int64_t T, int64_t D, int64_t P,
                      double *S, int nthreads)
{
    if (qko_check(x, dtype, T, D, P) != 0 || (T > 0 && S == NULL))
        return -1;
    if (nthreads <= 0)
        nthreads = 1;
    const size_t es = qko_elem_size(dtype);
#pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const char *row = (const char *)x + (size_t)t * (size_t)D * es;
        qko_row_partials(row, dtype, D, P, S + t * P);
    }
    return 0;
}

/*
 * y[t*D + j] and r[t] as defined above. y or r may be NULL when not wanted.
 * The P shard sums of a row are formed first, then added in order of p,
 * which is the order of Algorithm 1.
 */
int qko_rmsnorm(const void *x, int dtype, const float *gamma, int64_t T, int64_t D,
                int64_t P, double eps, double *y, double *r, int nthreads)
{
    if (qko_check(x, dtype, T, D, P) != 0 || gamma == NULL || !(eps >= 0.0))
        return -1;
    if (nthreads <= 0)
        nthreads = 1;
    const size_t es = qko_elem_size(dtype);
#pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const char *row = (const char *)x + (size_t)t * (size_t)D * es;
        double S = 0.0;
        /* Phase A, shard by shard, then the scalar sum over shards. */
        int64_t w = D / P;
        for (int64_t p = 0; p < P; ++p) {
            double s = 0.0;
            for (int64_t j = p * w; j < p * w + w; ++j) {
                double v = qko_load(row, dtype, j);
                s += v * v;
            }
            S += s;
        }
        /* Phase B: the factor, with the mean over the full width D. */
        double m = S / (double)D;
        double rt = 1.0 / sqrt(m + eps);
        if (r != NULL)
            r[t] = rt;
        /* Phase B weight multiply, then Phase C. */
        if (y != NULL) {
            for (int64_t j = 0; j < D; ++j) {
                double u = qko_load(row, dtype, j) * (double)gamma[j];
                y[t * D + j] = u * rt;
            }
        }
    }
    return 0;
}

/*
 * u[t*D + j] = x[t,j] * gamma[j] in double: the weight multiply on its own,
 * with no normalisation. This is what a deferred normalisation stores when a
 * later RMSNorm cancels the per-token factor ("perf(dsv4 decode swa):
 * deferred attention RMSNorm" pull request, attn_norm_xgamma), and it is
 * Algorithm 1's Phase B compute path by itself.
 */
int qko_xgamma(const void *x, int dtype, const float *gamma, int64_t T, int64_t D, double *u,
               int nthreads)
{
    if (qko_check(x, dtype, T, D, 1) != 0 || gamma == NULL || (T > 0 && u == NULL))
        return -1;
    if (nthreads <= 0)
        nthreads = 1;
    const size_t es = qko_elem_size(dtype);
#pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const char *row = (const char *)x + (size_t)t * (size_t)D * es;
        for (int64_t j = 0; j < D; ++j)
            u[t * D + j] = qko_load(row, dtype, j) * (double)gamma[j];
    }
    return 0;
}

/* 1 if built with OpenMP (the thread count is honoured), else 0. */
int qko_has_openmp(void)
{
#ifdef _OPENMP
    return 1;
#else
    return 0;
#endif
}
