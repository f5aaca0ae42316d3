/*
 * qknorm_oracle.c -- float64 CPU oracle for QK-Norm.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library.  The product
 * path (the CUDA library and its Python binding) never calls it, and the two
 * share no code, headers or helpers.
 *
 * What it computes (plain definitions, no blocking, no fusion):
 *
 *   RMSNorm of a vector x of length L with weight g and epsilon eps:
 *       m   = (1/L) * sum_j x_j^2
 *       y_j = x_j * g_j / sqrt(m + eps)
 *   "SwiftQK" review (pith.science verdict for arXiv 2608.09160),
 *   fields core_discovery and key_machinery: the divisor is
 *   sqrt(S_global/H + eps) with S_global = sum_j x_j^2 over the full vector.
 *
 *   Per-head QK-Norm (sglang PR #13189 "Add turbomind_rms_norm to accelerate
 *   QK norm in Qwen3 models", Motivation and Modifications): the RMSNorm
 *   module has hidden_size = head_dim, so every (token, head) row of length
 *   D is normalised on its own, with one weight g_q[D] for all query heads
 *   and one g_k[D] for all key heads.
 *
 *   Layerwise QK-Norm (SwiftQK abstract, newx.sg paper page): the
 *   normalisation factor depends on the full hidden vector, so per token the
 *   whole q vector (Hq*D elements) and the whole k vector (Hk*D elements)
 *   are each one RMSNorm row, with weights g_q[Hq*D] and g_k[Hk*D].
 *
 *   Sharded layerwise (SwiftQK review, key_machinery): each tensor-parallel
 *   rank r holds a contiguous head-aligned slice of the vector (split by head,
 *   "combined QKV projection" lesson, tensor-parallel follow-up question),
 *   computes S_r = sum of x_j^2 over its slice, and the ranks combine the
 *   scalars S = sum_r S_r; the divisor then uses the FULL length H, never the
 *   shard length.  Here the partials and the combine are in float64; this
 *   function exists to pin the decomposition, not to mimic float32.
 *
 * Buffer layout (the "combined QKV projection" lesson, GQA section): a fused
 * row-major activation [T, row_stride] whose columns [0, Hq*D) are Q,
 * [Hq*D, (Hq+Hk)*D) are K, then V (Hk*D columns), then padding up to
 * row_stride.  Every output element that is not Q or K is copied through
 * unchanged.
 *
 * Inputs are the stored bf16/fp32 values already widened (exactly) to
 * double by the caller; outputs are double.  Sums are sequential in index
 * order.  Token rows are independent; when nthreads > 1 an OpenMP loop over
 * tokens spreads them across host cores, which changes no arithmetic.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* RMSNorm of one row: y[j] = x[j] * g[j] / sqrt(sum(x^2)/L + eps). */
static void rmsnorm_row(const double *x, double *y, const double *g, int64_t L, double eps)
{
    double s = 0.0;
    for (int64_t j = 0; j < L; ++j) s += x[j] * x[j];
    const double m = s / (double)L;
    const double denom = sqrt(m + eps);
    for (int64_t j = 0; j < L; ++j) y[j] = x[j] * g[j] / denom;
}

static void copy_through(const double *x, double *y, int64_t T, int64_t row_stride)
{
    memcpy(y, x, (size_t)(T * row_stride) * sizeof(double));
}

static void set_threads(int nthreads)
{
#ifdef _OPENMP
    omp_set_num_threads(nthreads > 0 ? nthreads : 1);
#else
    (void)nthreads;
#endif
}

/* Per-head QK-Norm over every (token, head) row of length D. */
void oracle_per_head(const double *x, double *y, int64_t T, int Hq, int Hk, int D,
                     int64_t row_stride, const double *gamma_q, const double *gamma_k,
                     double eps, int nthreads)
{
    copy_through(x, y, T, row_stride);
    set_threads(nthreads);
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int h = 0; h < Hq + Hk; ++h) {
            const int64_t off = t * row_stride + (int64_t)h * D;
            const double *g = (h < Hq) ? gamma_q : gamma_k;
            rmsnorm_row(x + off, y + off, g, D, eps);
        }
    }
}

/* Layerwise QK-Norm: one row per token for q (Hq*D) and one for k (Hk*D). */
void oracle_layerwise(const double *x, double *y, int64_t T, int Hq, int Hk, int D,
                      int64_t row_stride, const double *gamma_q, const double *gamma_k,
                      double eps, int nthreads)
{
    copy_through(x, y, T, row_stride);
    set_threads(nthreads);
    const int64_t Lq = (int64_t)Hq * D, Lk = (int64_t)Hk * D;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const int64_t off = t * row_stride;
        if (Lq > 0) rmsnorm_row(x + off, y + off, gamma_q, Lq, eps);
        if (Lk > 0) rmsnorm_row(x + off + Lq, y + off + Lq, gamma_k, Lk, eps);
    }
}

/* One vector of length L split into nshards contiguous slices of L/nshards:
 * per-slice partial sums of squares, a combine of the scalars only, then the
 * full-length mean. */
static void sharded_row(const double *x, double *y, const double *g, int64_t L, int nshards,
                        double eps)
{
    const int64_t Ls = L / nshards;
    double S = 0.0;
    for (int r = 0; r < nshards; ++r) {
        double Sr = 0.0;
        for (int64_t j = r * Ls; j < (r + 1) * Ls; ++j) Sr += x[j] * x[j];
        S += Sr;
    }
    const double denom = sqrt(S / (double)L + eps);
    for (int64_t j = 0; j < L; ++j) y[j] = x[j] * g[j] / denom;
}

/* Layerwise QK-Norm with the scalar-statistics decomposition over nshards
 * head-aligned shards.  Returns 0, or -1 when nshards < 1 or does not divide
 * both Hq and Hk (a shard must hold whole heads). */
int oracle_layerwise_sharded(const double *x, double *y, int64_t T, int Hq, int Hk, int D,
                             int64_t row_stride, const double *gamma_q, const double *gamma_k,
                             double eps, int nshards, int nthreads)
{
    if (nshards < 1 || Hq % nshards != 0 || Hk % nshards != 0) return -1;
    copy_through(x, y, T, row_stride);
    set_threads(nthreads);
    const int64_t Lq = (int64_t)Hq * D, Lk = (int64_t)Hk * D;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const int64_t off = t * row_stride;
        if (Lq > 0) sharded_row(x + off, y + off, gamma_q, Lq, nshards, eps);
        if (Lk > 0) sharded_row(x + off + Lq, y + off + Lq, gamma_k, Lk, nshards, eps);
    }
    return 0;
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
