/*
 * row_softmax.h -- C ABI of the standalone row-wise softmax (B200, sm_100a).
 *
 * The operation: the fused-softmax step of "Designing High-Performance GPU Kernels
 * with TileLang" (pro.edgex.exchange summary, fused-softmax paragraph: max and sum
 * reductions over a row kept in registers), for every row r of a rows x n matrix:
 *
 *     y[r, j] = exp(x[r, j] - m_r) / sum_k exp(x[r, k] - m_r),   m_r = max_k x[r, k]
 *
 * The pages fix no layout or precision; the choices below are this library's.
 *
 * Layout: x and y rows x n, contiguous row-major, one dtype for both: ATTN_F16,
 * ATTN_BF16 (attn_fwd.h) or SOFTMAX_F32.  Arithmetic: fp32 (exp of x - m_r, fp32 sum),
 * y rounded once to its dtype.  Domain: finite x.
 *
 * Ownership: the caller owns x and y; the library allocates nothing and keeps no
 * pointer.  Asynchronous on `stream`.  y may be x itself (in place); any other
 * overlap is ATTN_ERR_ALIAS.
 *
 * Errors (codes of attn_fwd.h), returned before any CUDA call: ATTN_ERR_SHAPE (rows
 * < 0, n < 1 or n > ROW_SOFTMAX_MAX_N), ATTN_ERR_DTYPE, ATTN_ERR_NULLPTR (x or y
 * null with rows > 0), ATTN_ERR_ALIGN (x or y not aligned to its element size),
 * ATTN_ERR_ALIAS; then ATTN_ERR_DEVICE (no sm_100 device) or ATTN_ERR_LAUNCH.
 * rows == 0 is a no-op returning ATTN_OK.
 */
#ifndef ROW_SOFTMAX_H
#define ROW_SOFTMAX_H

#include "attn_fwd.h"

#ifdef __cplusplus
extern "C" {
#endif

/* dtype code of fp32 rows (ATTN_F16 = 0 and ATTN_BF16 = 1 come from attn_fwd.h) */
#define SOFTMAX_F32 2

/* Longest row accepted. */
#define ROW_SOFTMAX_MAX_N (1 << 28)

/*
 * row_softmax -- y = softmax(x) along each row.
 *   x      device, rows x n, dtype elements, aligned to the element size
 *   y      device, rows x n, same dtype, written; may equal x
 *   rows   >= 0;  n   1 .. ROW_SOFTMAX_MAX_N
 *   dtype  ATTN_F16, ATTN_BF16 or SOFTMAX_F32
 * Rows whose byte length is a multiple of 16 (with x, y 16-byte aligned) take the
 * vectorised paths; others a two-pass path.  Returns ATTN_OK once queued.
 */
int row_softmax(const void *x, void *y, long long rows, int n, int dtype,
                attn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* ROW_SOFTMAX_H */
