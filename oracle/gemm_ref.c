/*
 * gemm_ref.c -- plain fp64 CPU oracle for the GEMM with a fused bias + activation
 * epilogue.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file: only the tests and the CPU-baseline leg of the benchmark do.  It shares
 * no code, header, table or helper with the CUDA kernels.
 *
 * What it computes, with no blocking and no reordering beyond the definition, for
 * A [M,K], W [N,K] (both row-major) and bias [N]:
 *
 *   z[m,n] = sum_k A[m,k] * W[n,k]  (+ bias[n])
 *   C[m,n] = act(z[m,n]),  act = identity, GELU or ReLU
 *   GELU(z) = z * Phi(z) = 0.5 * z * (1 + erf(z / sqrt(2)))     (the exact form)
 *   ReLU(z) = max(z, 0)
 *
 * Source: "Designing High-Performance GPU Kernels with TileLang" as summarised on
 * pro.edgex.exchange (the tiled tensor-core GEMM with a fused bias + GELU epilogue)
 * and comrad404.com (the GEMM step, whose epilogue it names as a ReLU or a bias): the
 * two summaries disagree on the activation, so both are options here.  The pages
 * give neither the GELU form nor the layout: the exact (erf) GELU and W stored
 * [N,K] (C = A W^T, the layout of a linear layer's weight) are this library's
 * readings.
 *
 * Layouts: all row-major fp64.  OpenMP over rows of C.
 */
#include <math.h>

#ifdef _OPENMP
#include <omp.h>
#endif

enum { GEMM_REF_OK = 0, GEMM_REF_ERR_ARGS = 1 };
enum { ACT_NONE = 0, ACT_GELU = 1, ACT_RELU = 2 };

int gemm_ref_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static double activate(double z, int act)
{
    if (act == ACT_GELU)
        return 0.5 * z * (1.0 + erf(z / sqrt(2.0)));
    if (act == ACT_RELU)
        return z > 0.0 ? z : 0.0;
    return z;
}

/* bias may be NULL (no bias). */
int gemm_bias_act_ref_f64(const double *a, const double *w, const double *bias, double *c,
                          long M, long N, long K, int act)
{
    if (!a || !w || !c || M < 0 || N < 0 || K < 0 || act < ACT_NONE || act > ACT_RELU)
        return GEMM_REF_ERR_ARGS;
#pragma omp parallel for schedule(static)
    for (long m = 0; m < M; ++m) {
        for (long n = 0; n < N; ++n) {
            double z = 0.0;
            for (long k = 0; k < K; ++k)
                z += a[m * K + k] * w[n * K + k];
            if (bias)
                z += bias[n];
            c[m * N + n] = activate(z, act);
        }
    }
    return GEMM_REF_OK;
}
