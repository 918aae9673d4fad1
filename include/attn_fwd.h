/*
 * attn_fwd.h -- C ABI of the B200 (sm_100a) fused attention forward pass.
 *
 * The operation ("Designing High-Performance GPU Kernels with TileLang"; the
 * FlashAttention paragraph of the pro.edgex.exchange summary and "Cosa copre il
 * tutorial" on datastack.it): for every batch b, head h and query row i,
 *
 *     s_ij   = scale * sum_d Q[b,h,i,d] K[b,h,j,d]
 *     s_ij   = -inf  when causal and j > i          (top-left aligned mask)
 *     O[b,h,i,:] = sum_j softmax_j(s_i.) V[b,h,j,:]
 *     LSE[b,h,i] = ln sum_j exp(s_ij)                (natural log, scaled scores)
 *
 * computed tile by tile with an online softmax so the Sq x Sk score matrix never
 * reaches device memory.  The pages fix neither the layout, the mask alignment
 * for Sq != Sk, nor the log-sum-exp output; the choices below are this library's.
 *
 * Layout: Q [B,H,Sq,D], K and V [B,H,Sk,D], O [B,H,Sq,D], all contiguous
 * row-major 16-bit (one dtype for all four); LSE [B,H,Sq] contiguous fp32.
 * Arithmetic: 16-bit operands, fp32 accumulation and softmax, one rounding of O.
 *
 * Ownership: the caller owns every buffer.  The library allocates no memory and
 * keeps no pointer after a call returns.  Device-pointer calls are asynchronous on
 * `stream` (the stream's previous work completes first; nothing else is
 * synchronised).
 *
 * Errors: argument errors return a negative code before any CUDA call and leave
 * every buffer untouched.  A failed launch returns ATTN_ERR_LAUNCH.  A kernel whose
 * pipeline wait runs out of time (2 s per wait) stops, records ATTN_ERR_TIMEOUT in
 * the per-device status word (read it with attn_fwd_status) and leaves O / LSE
 * undefined; nothing traps or aborts.
 */
#ifndef ATTN_FWD_H
#define ATTN_FWD_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; a null stream is the legacy default stream. */
typedef struct CUstream_st *attn_stream_t;

/* Element type of Q, K, V and O. */
typedef enum { ATTN_F16 = 0, ATTN_BF16 = 1 } attn_dtype_t;

/* Mask of attn_fwd_ex.  ATTN_MASK_CAUSAL is the `causal` of attn_fwd: key j visible to
 * query i iff j <= i (top-left).  ATTN_MASK_CAUSAL_BOTTOM_RIGHT: iff j <= i + Sk - Sq
 * (the last query sees every key); with Sq > Sk the first Sq - Sk query rows see no key
 * and get O = 0, LSE = -inf. */
typedef enum {
    ATTN_MASK_NONE = 0,
    ATTN_MASK_CAUSAL = 1,
    ATTN_MASK_CAUSAL_BOTTOM_RIGHT = 2
} attn_mask_t;

enum {
    ATTN_OK = 0,
    ATTN_ERR_NULLPTR = -1,   /* q, k, v or o is null                                */
    ATTN_ERR_ALIGN = -2,     /* q, k, v, o not 16-byte aligned, or lse not 4-byte   */
    ATTN_ERR_SHAPE = -3,     /* B, H, Sq or Sk < 1, or a size beyond the limits     */
    ATTN_ERR_HEADDIM = -4,   /* D is not 64, 80, 96, 112, 128, 192 or 256           */
    ATTN_ERR_DTYPE = -5,     /* dtype is not ATTN_F16 / ATTN_BF16                   */
    ATTN_ERR_TENSORMAP = -6, /* the driver refused a TMA descriptor                 */
    ATTN_ERR_LAUNCH = -7,    /* a CUDA call or the kernel launch failed             */
    ATTN_ERR_TIMEOUT = -8,   /* (status word) a pipeline wait ran out of time       */
    ATTN_ERR_SCALE = -9,     /* scale is NaN or infinite                            */
    ATTN_ERR_ALIAS = -10,    /* o or lse overlaps q, k or v                         */
    ATTN_ERR_DEVICE = -11,   /* no CUDA device, or the current one is not sm_100    */
    ATTN_ERR_WORKSPACE = -12,/* split pass: workspace smaller than required         */
    ATTN_ERR_MASK = -13      /* attn_fwd_ex: mask is not an ATTN_MASK_* value       */
};

/*
 * attn_fwd -- O and LSE from device buffers.
 *   q      device, [B,H,Sq,D] 16-bit, 16-byte aligned
 *   k, v   device, [B,H,Sk,D] 16-bit, 16-byte aligned
 *   o      device, [B,H,Sq,D] 16-bit, 16-byte aligned, written; must not overlap q/k/v
 *   lse    device, [B,H,Sq] fp32, written; may be NULL (not written)
 *   B, H, Sq, Sk >= 1; B*H, Sq, Sk <= 2^24; D in {64, 80, 96, 112, 128, 192, 256}
 *          (80, 96 and 112 run as 128 with the missing columns read as zeros: exact, at
 *          the cost of the padded work; 192 and 256 run on pairs of CTAs that share
 *          each MMA, or, for at most 128 query rows per K/V head, in a kernel with
 *          128-row query tiles and 64-key K/V tiles)
 *   causal 0: every key visible; nonzero: key j visible to query i iff j <= i
 *   scale  finite multiplier of q.k (e.g. 1/sqrt(D)); |scale*q.k| must fit fp32
 *   dtype  ATTN_F16 or ATTN_BF16
 *   stream the CUDA stream to run on
 * Returns ATTN_OK once the kernel is queued, or a negative code (see above).
 */
int attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
             int B, int H, int Sq, int Sk, int D, int causal, float scale,
             int dtype, attn_stream_t stream);

/*
 * attn_fwd_host -- the same pass from host buffers: copies q, k, v host -> device
 * staging buffers, runs attn_fwd, copies o (and lse when both lse pointers are
 * non-null) back, all ordered on `stream`; the caller synchronises the stream before
 * reading o_host / lse_host.  Host buffers should be page-locked for the copies to
 * be asynchronous.  The staging buffers (q_dev ... lse_dev) are caller-allocated
 * device memory with the shapes and alignment attn_fwd requires.
 * A pass of at least 16 MB of q, k and v runs as up to 8 chunks of whole heads in a
 * pipeline: a chunk's inputs are copied in on one of the library's copy streams while
 * the previous chunk's pass runs on `stream` and the chunk before it is copied out on
 * the other, so both directions of the host link and the kernel overlap.  The two
 * copy streams (non-blocking) and four events are created on the current device at
 * the first such call and kept for the life of the process (not valid across
 * cudaDeviceReset); every copy is joined back into `stream` before the call returns,
 * on error paths too, so that `stream` orders all of the call's work and a capture of
 * `stream` into a graph stays joined.  Concurrent calls on one device queue their
 * chunks one call after the other.
 */
int attn_fwd_host(const void *q_host, const void *k_host, const void *v_host,
                  void *o_host, float *lse_host,
                  void *q_dev, void *k_dev, void *v_dev, void *o_dev, float *lse_dev,
                  int B, int H, int Sq, int Sk, int D, int causal, float scale,
                  int dtype, attn_stream_t stream);

/*
 * attn_fwd_splitkv -- the same pass computed as n_splits independent KV ranges per
 * (256-row query block, head), for shapes with few query rows and long key sequences
 * (decoding): each range writes its own normalised partial O and log-sum-exp into
 * `workspace` (fp32), and a second kernel merges them,
 *     LSE = ln sum_s exp(LSE_s),   O = sum_s exp(LSE_s - LSE) O_s,
 * which is the whole-range softmax attention exactly (each range's weight is its share
 * of the full normaliser; a range no key of which a row sees has LSE_s = -inf).  The
 * pages describe the online-softmax rescaling this relies on; the split itself is this
 * library's (no counterpart on the pages).
 *   n_splits   1 .. 1024 ranges of ceil(ceil(Sk/T) / n_splits) T-key tiles each, T = 128
 *              (T = 64 for D = 192 / 256 with at most 128 query rows, the decode shapes
 *              of the wide kernel); trailing ranges may be empty;
 *              attn_fwd_splitkv_default_splits picks one for the device
 *   workspace  device, 256-byte aligned, at least attn_fwd_splitkv_workspace_bytes(B,
 *              H, Sq, D, n_splits) bytes, caller-owned, not overlapping any argument;
 *              its contents are scratch (overwritten each call)
 * Other arguments, layouts and errors as attn_fwd; ATTN_ERR_WORKSPACE when the
 * workspace is too small.  Two kernels are queued on `stream`.
 */
int attn_fwd_splitkv(const void *q, const void *k, const void *v, void *o, float *lse,
                     int B, int H, int Sq, int Sk, int D, int causal, float scale,
                     int dtype, int n_splits, void *workspace, size_t workspace_bytes,
                     attn_stream_t stream);

/*
 * attn_fwd_ex -- the general entry point: grouped K/V heads, the mask choice and the
 * split-KV option in one call (attn_fwd and attn_fwd_splitkv are special cases).
 *   H_kv   heads of K and V, a divisor of H: k, v are [B,H_kv,Sk,D] and query head h
 *          reads K/V head h / (H / H_kv) (grouped-query attention; H_kv = H is plain
 *          multi-head attention).  The H / H_kv query heads of a group are processed
 *          together as one sequence of (H / H_kv) * Sq rows, which must be <= 2^24.
 *   mask   ATTN_MASK_NONE, ATTN_MASK_CAUSAL or ATTN_MASK_CAUSAL_BOTTOM_RIGHT
 *          (ATTN_ERR_MASK otherwise)
 *   n_splits  0: the whole pass (workspace may be NULL); 1 .. 1024: the split pass
 *          with `workspace` as for attn_fwd_splitkv (its size from
 *          attn_fwd_splitkv_workspace_bytes(B, H, Sq, D, n_splits))
 * The pages name causal and non-causal attention only; grouped heads and the
 * bottom-right alignment are this library's options.
 */
int attn_fwd_ex(const void *q, const void *k, const void *v, void *o, float *lse,
                int B, int H, int H_kv, int Sq, int Sk, int D, int mask, float scale,
                int dtype, int n_splits, void *workspace, size_t workspace_bytes,
                attn_stream_t stream);

/* attn_fwd_splitkv_default_splits for attn_fwd_ex's arguments (0 for invalid ones). */
int attn_fwd_ex_default_splits(int B, int H, int H_kv, int Sq, int Sk, int D, int mask);

/* Bytes of workspace attn_fwd_splitkv needs (0 for invalid arguments). */
size_t attn_fwd_splitkv_workspace_bytes(int B, int H, int Sq, int D, int n_splits);

/* A split count for these sizes on the current device: the one that balances
 * (query block, head, range) units over the SMs best, counted in the geometry of the
 * kernel that runs D (its query rows and keys per tile, and two SMs per unit on the
 * D = 192 / 256 CTA pairs) (1 .. 1024; 0 for invalid sizes). */
int attn_fwd_splitkv_default_splits(int B, int H, int Sq, int Sk, int D, int causal);

/* Size of the scratch attn_fwd_splitkv_noalloc uses in place of a workspace. */
#define ATTN_SPLITKV_NOALLOC_SCRATCH_BYTES (16u << 20)

/*
 * attn_fwd_splitkv_noalloc -- attn_fwd_splitkv for callers that must not allocate
 * device memory for the call and cannot hand over a workspace of their own: a
 * serving loop whose device memory is all reserved at start-up, or a plain C caller
 * with no device allocator at hand.  The partial results go to a scratch array of
 * ATTN_SPLITKV_NOALLOC_SCRATCH_BYTES that the library keeps in its own static device
 * memory, one per device; nothing is allocated per call.  (The split-KV merge is this
 * library's; the pages have no counterpart of it or of this entry point.)
 *   Arguments, layouts and results as attn_fwd_splitkv, without the workspace.
 *   ATTN_ERR_WORKSPACE when attn_fwd_splitkv_workspace_bytes(B, H, Sq, D, n_splits)
 *   exceeds ATTN_SPLITKV_NOALLOC_SCRATCH_BYTES (use attn_fwd_splitkv, or fewer
 *   splits); no CUDA call is made then.
 *   The scratch needs no initialisation: every value the merge reads is written by
 *   the same call first.
 *   The first call on a device looks up the scratch's device address (one runtime
 *   call, which may load the library's device code on that device) and keeps it;
 *   make that first call before any stream capture begins.
 *   One scratch per device: calls on one device that can overlap (different streams,
 *   or threads without ordering) race on it and give undefined results.  Calls
 *   ordered on one stream are safe.
 *   The looked-up address (like the library's other per-device set-up: kernel
 *   attributes, cluster occupancy) is kept for the life of the process and is not
 *   valid across cudaDeviceReset: a process that resets a device must not call this
 *   library on that device again.
 */
int attn_fwd_splitkv_noalloc(const void *q, const void *k, const void *v, void *o, float *lse,
                             int B, int H, int Sq, int Sk, int D, int causal, float scale,
                             int dtype, int n_splits, attn_stream_t stream);

/*
 * attn_fwd_status -- synchronise `stream`, copy the current device's status word
 * into *device_status (0, or the first ATTN_ERR_* a kernel of this library -- the
 * attention kernels, then the GEMM kernels of gemm_bias_act.h -- recorded since the
 * last read) and reset it to 0.  Returns ATTN_OK, ATTN_ERR_NULLPTR or ATTN_ERR_LAUNCH.
 */
int attn_fwd_status(attn_stream_t stream, int *device_status);

/* Static string naming an ATTN_* code (never NULL). */
const char *attn_fwd_strerror(int code);

/* ABI version of this header, currently 2 (the split-count helpers take D). */
int attn_fwd_abi_version(void);

/*
 * attn_fwd_debug -- attn_fwd with debug flags, for the tests.  Flag 1 makes the TMA
 * producer skip the Q load so the MMA warp's first wait runs out: the call must end
 * with ATTN_ERR_TIMEOUT in the status word, not hang.  Flag 2 (host side only) makes
 * the TMA descriptor encoding report failure: the call returns ATTN_ERR_TENSORMAP
 * and launches nothing.  Flag 0 is attn_fwd.
 */
int attn_fwd_debug(const void *q, const void *k, const void *v, void *o, float *lse,
                   int B, int H, int Sq, int Sk, int D, int causal, float scale,
                   int dtype, attn_stream_t stream, unsigned flags);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_FWD_H */
