/*
 * gemm_bias_act.h -- C ABI of the GEMM with a fused bias + activation epilogue
 * (B200, sm_100a tensor cores).
 *
 * The operation: the tiled tensor-core GEMM of "Designing High-Performance GPU
 * Kernels with TileLang" with its fused epilogue (pro.edgex.exchange summary: bias +
 * GELU; comrad404.com summary, "Как устроен туториал": ReLU or bias -- the two
 * summaries differ, so both activations are offered):
 *
 *     C[m, n] = act( sum_k A[m, k] * W[n, k]  +  bias[n] )
 *     act = identity, GELU(z) = 0.5 z (1 + erf(z / sqrt 2)) (the exact form), or ReLU
 *
 * The pages fix no layout; W is stored [N, K] (C = A W^T, a linear layer's weight).
 *
 * Layout: A [M, K], W [N, K], C [M, N], contiguous row-major, bias [N] (or NULL), all
 * one 16-bit dtype (ATTN_F16 / ATTN_BF16 of attn_fwd.h).  Arithmetic: 16-bit products
 * accumulated in fp32 on the tensor cores; bias and activation in fp32; C rounded once.
 * Requirements: M, N, K >= 1; N and K multiples of 8; A, W, C 16-byte aligned, bias
 * 2-byte aligned; C must not overlap A, W or bias.
 *
 * Ownership: the caller owns every buffer; the library allocates nothing and keeps no
 * pointer.  Asynchronous on `stream`.
 *
 * Errors (codes of attn_fwd.h), returned before any CUDA call: ATTN_ERR_NULLPTR,
 * ATTN_ERR_DTYPE, ATTN_ERR_SHAPE (sizes, or act not a GEMM_ACT_* value),
 * ATTN_ERR_ALIGN, ATTN_ERR_ALIAS; then ATTN_ERR_DEVICE, ATTN_ERR_TENSORMAP or
 * ATTN_ERR_LAUNCH.  A pipeline wait that runs out of time (2 s) ends the kernel and
 * records ATTN_ERR_TIMEOUT in the status word that attn_fwd_status reads.
 */
#ifndef GEMM_BIAS_ACT_H
#define GEMM_BIAS_ACT_H

#include "attn_fwd.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { GEMM_ACT_NONE = 0, GEMM_ACT_GELU = 1, GEMM_ACT_RELU = 2 } gemm_act_t;

/*
 * gemm_bias_act -- C = act(A W^T + bias).
 *   a     device, [M, K];  w  device, [N, K];  bias  device, [N] or NULL (no bias)
 *   c     device, [M, N], written
 *   act   GEMM_ACT_NONE, GEMM_ACT_GELU or GEMM_ACT_RELU
 *   dtype ATTN_F16 or ATTN_BF16 (all four buffers)
 * Returns ATTN_OK once the kernel is queued, or a negative code.
 */
int gemm_bias_act(const void *a, const void *w, const void *bias, void *c, int M, int N,
                  int K, int act, int dtype, attn_stream_t stream);

/*
 * gemm_bias_act_debug -- gemm_bias_act with kernel debug flags, for the tests.  Flag 1
 * makes the TMA producer skip its loads so the MMA warp's first wait runs out: the
 * call must end with ATTN_ERR_TIMEOUT in the status word, not hang.  Flag 2 forces the
 * 128-row output tiles, flag 4 the 256-row tiles (gemm_bias_act picks by K).  Flag 0
 * is gemm_bias_act.
 */
int gemm_bias_act_debug(const void *a, const void *w, const void *bias, void *c, int M,
                        int N, int K, int act, int dtype, attn_stream_t stream,
                        unsigned flags);

#ifdef __cplusplus
}
#endif

#endif /* GEMM_BIAS_ACT_H */
