/*
 * softmax_ref.c -- plain fp64 CPU oracle for the row-wise softmax.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file: only the tests and the CPU-baseline leg of the benchmark do.  It shares
 * no code, header, table or helper with the CUDA kernels.
 *
 * What it computes (the definition, with no blocking, no online rescaling, no
 * fusion), for every row r of a rows x n matrix:
 *
 *   m_r    = max_j x[r,j]
 *   y[r,j] = exp(x[r,j] - m_r) / sum_k exp(x[r,k] - m_r)
 *
 * Source: "Designing High-Performance GPU Kernels with TileLang" as summarised on
 * pro.edgex.exchange (the fused-softmax paragraph: a row-wise softmax whose max and
 * sum reductions stay in registers) and comrad404.com ("Как устроен туториал": the
 * softmax step between the GEMM and FlashAttention parts).  Subtracting the row max
 * changes nothing mathematically (the factor exp(-m_r) cancels); it keeps exp from
 * overflowing.  Domain: finite inputs, n >= 1.
 *
 * Every row is checked to sum to one within 1e-12 + n * 2^-52, the rounding bound of
 * an n-term fp64 sum (ORACLE_ERR_ROWSUM otherwise).
 * Layout: x and y rows x n, contiguous row-major fp64.  OpenMP over rows.
 */
#include <float.h>
#include <math.h>
#include <stdlib.h>

#ifdef _OPENMP
#include <omp.h>
#endif

enum { SOFTMAX_OK = 0, SOFTMAX_ERR_ARGS = 1, SOFTMAX_ERR_ROWSUM = 3 };

int softmax_ref_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* One row: max, exponentials, normaliser, division. */
static int softmax_one_row(const double *x, double *y, long n)
{
    double m = -INFINITY;
    for (long j = 0; j < n; ++j)
        if (x[j] > m)
            m = x[j];
    double l = 0.0;
    for (long j = 0; j < n; ++j) {
        y[j] = exp(x[j] - m);
        l += y[j];
    }
    double total = 0.0;
    for (long j = 0; j < n; ++j) {
        y[j] = y[j] / l;
        total += y[j];
    }
    /* a sum of n fp64 terms of total 1 is off by at most (n - 1) * 2^-53 */
    return fabs(total - 1.0) <= 1e-12 + (double)n * DBL_EPSILON ? SOFTMAX_OK
                                                                 : SOFTMAX_ERR_ROWSUM;
}

int softmax_ref_f64(const double *x, double *y, long rows, long n)
{
    if (!x || !y || rows < 0 || n < 1)
        return SOFTMAX_ERR_ARGS;
    int status = SOFTMAX_OK;
#pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; ++r) {
        int rc = softmax_one_row(x + r * n, y + r * n, n);
        if (rc != SOFTMAX_OK) {
#pragma omp atomic write
            status = rc;
        }
    }
    return status;
}
