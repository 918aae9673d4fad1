/*
 * attn_ref.c -- plain fp64 CPU oracle for the fused attention forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file: only the tests, the package smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header, table or helper with the CUDA
 * kernels.
 *
 * What it computes is the definition the tiled kernel must reach (up to floating
 * point rounding), written out with no blocking, no online rescaling and no
 * fusion:
 *
 *   s_ij   = scale * sum_d Q[i,d] K[j,d]                  scaled scores
 *   s_ij   = -inf         if causal and j > i + off       causal mask: off = 0 aligns
 *                                                         it top-left, off = Sk - Sq
 *                                                         bottom-right
 *   m_i    = max_j s_ij
 *   p_ij   = exp(s_ij - m_i) / sum_j exp(s_ij - m_i)      row softmax
 *   O[i,:] = sum_j p_ij V[j,:]
 *   LSE_i  = m_i + ln(sum_j exp(s_ij - m_i))              natural log of the row
 *                                                         normaliser of the scaled
 *                                                         scores
 *
 * Source: "Designing High-Performance GPU Kernels with TileLang" as summarised on
 * pro.edgex.exchange (the FlashAttention paragraph: the fused forward pass must give
 * the same softmax attention as PyTorch scaled-dot-product attention, causal and
 * non-causal, without storing the score matrix in global memory) and on datastack.it
 * ("Cosa copre il tutorial": causal and non-causal FlashAttention with online
 * softmax).  The pages give the method only in prose; the formula above is the plain
 * softmax attention they validate against.  Readings taken where the pages are
 * silent: the causal mask is top-left aligned (key j is visible to query i when
 * j <= i, the convention of PyTorch's is_causal); the log-sum-exp is the natural log
 * of the normaliser of the *scaled* scores.
 *
 * Every per-head score matrix (or, for the row entry point, every score row) is
 * materialised in fp64 before the softmax, with libm exp/log and no fast-math.
 * Each call checks, for every output row, that the softmax row sums to one within
 * 1e-12; a failed check returns ORACLE_ERR_ROWSUM.
 *
 * Extensions of the same definition (the pages name only causal and non-causal; these
 * are this library's options, written out the same plain way):
 *   - bottom-right causal alignment (off = Sk - Sq: the last query row sees every
 *     key); with Sq > Sk the first Sq - Sk rows then see no key at all, and such a
 *     row is defined as O = 0, LSE = -inf (the empty sum);
 *   - grouped K/V heads: Hkv divides H, query head h reads K/V head h / (H / Hkv).
 *
 * Layouts: Q [B,H,Sq,D], K and V [B,Hkv,Sk,D], O [B,H,Sq,D], LSE [B,H,Sq], all
 * contiguous row-major fp64.  Threads: OpenMP over heads (full entry point) or over
 * rows (row entry point).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* mask argument */
enum { ORACLE_NO_MASK = 0, ORACLE_CAUSAL_TOP_LEFT = 1, ORACLE_CAUSAL_BOTTOM_RIGHT = 2 };

enum {
    ORACLE_OK = 0,
    ORACLE_ERR_ARGS = 1,
    ORACLE_ERR_NOMEM = 2,
    ORACLE_ERR_ROWSUM = 3
};

/* Threads the OpenMP runtime will use for the parallel loops below. */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * One query row: fill srow[0..Sk) with the masked scaled scores of query i, turn it
 * into the softmax row in place, then write O[i,:] and LSE_i.
 * q_i: D values; kh, vh: the head's K and V, Sk x D.
 * Returns ORACLE_OK or ORACLE_ERR_ROWSUM.
 */
static int attend_one_row(const double *q_i, const double *kh, const double *vh,
                          long i, long Sq, long Sk, long D, int mask, double scale,
                          double *srow, double *o_i, double *lse_i)
{
    /* scores, then the causal mask */
    for (long j = 0; j < Sk; ++j) {
        double dot = 0.0;
        for (long d = 0; d < D; ++d)
            dot += q_i[d] * kh[j * D + d];
        srow[j] = scale * dot;
    }
    if (mask != ORACLE_NO_MASK) {
        const long off = (mask == ORACLE_CAUSAL_BOTTOM_RIGHT) ? Sk - Sq : 0;
        for (long j = (i + 1 + off > 0 ? i + 1 + off : 0); j < Sk; ++j)
            srow[j] = -INFINITY;
    }

    /* softmax over the row: max, exponentials, normaliser, division */
    double m = -INFINITY;
    for (long j = 0; j < Sk; ++j)
        if (srow[j] > m)
            m = srow[j];
    if (m == -INFINITY) {
        /* no visible key: the empty sum (no weights, O = 0, LSE = ln 0) */
        for (long j = 0; j < Sk; ++j)
            srow[j] = 0.0;
        for (long d = 0; d < D; ++d)
            o_i[d] = 0.0;
        *lse_i = -INFINITY;
        return ORACLE_OK;
    }
    double l = 0.0;
    for (long j = 0; j < Sk; ++j) {
        srow[j] = exp(srow[j] - m);
        l += srow[j];
    }
    double total = 0.0;
    for (long j = 0; j < Sk; ++j) {
        srow[j] = srow[j] / l;
        total += srow[j];
    }
    if (!(fabs(total - 1.0) <= 1e-12))
        return ORACLE_ERR_ROWSUM;

    /* probabilities times V */
    for (long d = 0; d < D; ++d)
        o_i[d] = 0.0;
    for (long j = 0; j < Sk; ++j) {
        const double pj = srow[j];
        const double *v_j = vh + j * D;
        for (long d = 0; d < D; ++d)
            o_i[d] += pj * v_j[d];
    }
    *lse_i = m + log(l);
    return ORACLE_OK;
}

static int shape_ok(long B, long H, long Hkv, long Sq, long Sk, long D, int mask)
{
    return B >= 1 && H >= 1 && Hkv >= 1 && H % Hkv == 0 && Sq >= 1 && Sk >= 1 && D >= 1 &&
           mask >= ORACLE_NO_MASK && mask <= ORACLE_CAUSAL_BOTTOM_RIGHT;
}

/* Index of the K/V head that query head h of batch b reads. */
static long kv_head(long b, long h, long H, long Hkv)
{
    return b * Hkv + h / (H / Hkv);
}

/*
 * Full problem.  For each (b, h) the Sq x Sk score matrix is materialised in fp64,
 * masked, softmaxed row by row, and multiplied by V.
 * p_out (nullable) receives the probability matrices, [B,H,Sq,Sk].
 */
int attn_ref_ex_f64(const double *q, const double *k, const double *v,
                    double *o, double *lse, double *p_out,
                    long B, long H, long Hkv, long Sq, long Sk, long D,
                    int mask, double scale)
{
    if (!q || !k || !v || !o || !lse || !shape_ok(B, H, Hkv, Sq, Sk, D, mask))
        return ORACLE_ERR_ARGS;

    const long heads = B * H;
    int status = ORACLE_OK;

#pragma omp parallel
    {
        double *smat = (double *)malloc(sizeof(double) * (size_t)Sq * (size_t)Sk);
        if (!smat) {
#pragma omp atomic write
            status = ORACLE_ERR_NOMEM;
        }
#pragma omp for schedule(dynamic, 1)
        for (long bh = 0; bh < heads; ++bh) {
            if (!smat)
                continue;
            const double *qh = q + bh * Sq * D;
            const long kvh = kv_head(bh / H, bh % H, H, Hkv);
            const double *kh = k + kvh * Sk * D;
            const double *vh = v + kvh * Sk * D;
            for (long i = 0; i < Sq; ++i) {
                int rc = attend_one_row(qh + i * D, kh, vh, i, Sq, Sk, D, mask, scale,
                                        smat + i * Sk, o + (bh * Sq + i) * D,
                                        lse + bh * Sq + i);
                if (rc != ORACLE_OK) {
#pragma omp atomic write
                    status = rc;
                }
            }
            if (p_out)
                memcpy(p_out + bh * Sq * Sk, smat, sizeof(double) * (size_t)Sq * (size_t)Sk);
        }
        free(smat);
    }
    return status;
}

/* The original entry point: K/V heads = query heads, causal = top-left. */
int attn_ref_f64(const double *q, const double *k, const double *v,
                 double *o, double *lse, double *p_out,
                 long B, long H, long Sq, long Sk, long D,
                 int causal, double scale)
{
    return attn_ref_ex_f64(q, k, v, o, lse, p_out, B, H, H, Sq, Sk, D,
                           causal ? ORACLE_CAUSAL_TOP_LEFT : ORACLE_NO_MASK, scale);
}

/*
 * Selected rows only (the same definition restricted to the requested query rows,
 * for spot checks of problems too large to run whole).
 * rows: n triples (b, h, i).  o: n x D, lse: n.
 */
int attn_ref_rows_ex_f64(const double *q, const double *k, const double *v,
                         const int64_t *rows, long n, double *o, double *lse,
                         long B, long H, long Hkv, long Sq, long Sk, long D,
                         int mask, double scale)
{
    if (!q || !k || !v || !rows || !o || !lse || n < 0 ||
        !shape_ok(B, H, Hkv, Sq, Sk, D, mask))
        return ORACLE_ERR_ARGS;
    for (long r = 0; r < n; ++r) {
        if (rows[3 * r] < 0 || rows[3 * r] >= B || rows[3 * r + 1] < 0 ||
            rows[3 * r + 1] >= H || rows[3 * r + 2] < 0 || rows[3 * r + 2] >= Sq)
            return ORACLE_ERR_ARGS;
    }

    int status = ORACLE_OK;
#pragma omp parallel
    {
        double *srow = (double *)malloc(sizeof(double) * (size_t)Sk);
        if (!srow) {
#pragma omp atomic write
            status = ORACLE_ERR_NOMEM;
        }
#pragma omp for schedule(dynamic, 4)
        for (long r = 0; r < n; ++r) {
            if (!srow)
                continue;
            const long bh = rows[3 * r] * H + rows[3 * r + 1];
            const long kvh = kv_head(rows[3 * r], rows[3 * r + 1], H, Hkv);
            const long i = rows[3 * r + 2];
            int rc = attend_one_row(q + (bh * Sq + i) * D, k + kvh * Sk * D, v + kvh * Sk * D,
                                    i, Sq, Sk, D, mask, scale, srow, o + r * D, lse + r);
            if (rc != ORACLE_OK) {
#pragma omp atomic write
                status = rc;
            }
        }
        free(srow);
    }
    return status;
}

int attn_ref_rows_f64(const double *q, const double *k, const double *v,
                      const int64_t *rows, long n, double *o, double *lse,
                      long B, long H, long Sq, long Sk, long D,
                      int causal, double scale)
{
    return attn_ref_rows_ex_f64(q, k, v, rows, n, o, lse, B, H, H, Sq, Sk, D,
                                causal ? ORACLE_CAUSAL_TOP_LEFT : ORACLE_NO_MASK, scale);
}
