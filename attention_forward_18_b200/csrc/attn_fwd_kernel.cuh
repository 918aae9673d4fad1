// attn_fwd_kernel.cuh -- fused attention forward pass for sm_100a (B200).
//
// O = softmax(scale * Q K^T [+ top-left causal mask]) V and the natural-log
// log-sum-exp per query row, computed tile by tile with an online softmax so the
// score matrix never reaches global memory ("Designing High-Performance GPU Kernels
// with TileLang", FlashAttention section of the pro.edgex.exchange summary: running
// row maxima, running normalisers, rescaling of the partial output, tiled
// tensor-core matrix products; comrad404.com "Финал": parallel over heads with
// sequential reads from HBM).
//
// Work unit: one CTA owns two 128-row query tiles (rows q0 .. q0+255) of one
// (batch, head) and streams that head's K/V in 128-key tiles; both query tiles share
// every K/V tile brought into shared memory.
//
//   warps 0-3   softmax of query tile 0 (thread t owns row t of the tile); also
//               rescales O_0 in TMEM on the rare KV tiles where a row max moved
//   warps 4-7   softmax of query tile 1 (same for O_1)
//   warps 8-11  epilogue: O / l, 16-bit rounding, stores of O and LSE
//   warp 12     MMA issuer (one thread)
//   warp 13     TMA producer (one thread)
//   warp 14     owns the tensor-memory allocation
//   warp 15     idle
//
// Tensor memory (512 columns): S_0 at 0, S_1 at 128 (fp32 scores, then the 16-bit
// probabilities P_t written over the first 64 columns), O_0 at 256, O_1 at 256 + D.
// The MMA thread ping-pongs the two tiles so one tile's softmax overlaps the other
// tile's matrix products:
//     S_0,0  S_1,0 | PV_0,0  S_0,1 | PV_1,0  S_1,1 | PV_0,1  S_0,2 | ...
// tcgen05 MMAs issued by one thread complete in issue order, so once S_t,j is
// complete PV_t,j-1 is too and nothing touches O_t until P_t,j is handed over: the
// softmax warps rescale O_t in place at that point, with no extra hand-off.
// Shared memory: Q_0, Q_1 and an NS-stage ring of K and of V tiles; each tile is
// 128 rows x D stored as D/64 column chunks of 128 rows x 128 bytes in the 128-byte
// swizzle that TMA writes and the tcgen05 smem descriptors read.
//
// Registers: 512 threads launch with 128 registers each; setmaxnreg moves them to
// 200 for the softmax warpgroups, 48 for the epilogue warpgroup and 64 for the
// MMA / TMA / allocator warps (2*128*200 + 128*48 + 128*64 = 65536).
//
// Every mbarrier wait is bounded (WAIT_LIMIT_NS); on expiry the waiting role records
// ATTN_ERR_TIMEOUT in the device status word and flags the CTA; every role then
// leaves its loop, waits (again bounded) for the copies / MMAs it started, and the
// CTA frees its tensor memory and exits.
#pragma once

#include <cuda.h>
#include <cstdint>

#include "ptx.cuh"

namespace attn {

constexpr int BM = 128;                 // query rows per tile (= TMEM lanes)
constexpr int BN = 128;                 // keys per tile
constexpr int ROWS_PER_CTA = 2 * BM;    // two query tiles per CTA
constexpr int CHUNK_ELEMS = 64;         // 16-bit elements per 128-byte swizzle row
constexpr int CHUNK_BYTES = 128 * 128;  // one chunk: 128 rows x 128 bytes
constexpr int NUM_THREADS = 512;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_S = 0;          // + 128 * tile
constexpr uint32_t TMEM_O = 256;        // + D * tile
// Lazy rescaling: the running max used for the exponentials only moves when a row's
// new max exceeds it by more than this (log2 units).  Until then P can reach 2^8,
// well inside fp16/bf16 range, and O and l stay consistent because both accumulate
// relative to the same (stale) max, so O / l is unchanged.
constexpr float LAZY_RESCALE_LOG2 = 8.0f;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;   // 2 s per wait
constexpr uint64_t DRAIN_LIMIT_NS = 500000000ull;   // 0.5 s per drain wait

constexpr int STATUS_TIMEOUT = -8;  // ATTN_ERR_TIMEOUT

// Bit 0: the producer never issues the Q loads, so the MMA thread's first wait runs
// out; only the timeout test sets it.
constexpr uint32_t FLAG_SKIP_Q_LOAD = 1u;

// Rows and heads as the kernel sees them: with grouped K/V heads (g query heads per
// K/V head) the g query heads of a group are adjacent in [B, H, Sq, D], so Q, O and
// LSE are read as [B*Hkv, g*Sq, ...] and one "head" of the kernel is a K/V head with
// g*Sq query rows; packed row r is query position r % sq_head.
struct Params {
    void* o;            // [BH, Sq, D] 16-bit (whole pass)
    float* lse;         // [BH, Sq] fp32, may be null (whole pass)
    float* ws_o;        // split-KV: [n_splits, BH, Sq, D] fp32 partial O (normalised)
    float* ws_lse;      // split-KV: [n_splits, BH, Sq] fp32 partial LSE
    int Sq, Sk, BH, n_qp;  // packed query rows, keys, K/V heads, 256-row query pairs
    int sq_head;        // query positions per query head (Sq / g)
    int d_out;          // head dimension of the tensors (<= D; Q, K, V read as zero-padded
                        // to D, O and the partials written for d_out columns)
    int causal_off;     // causal: key j visible to position i iff j <= i + causal_off
    int n_splits;       // KV ranges per (query pair, head); 1 for the whole pass
    int chunk_tiles;    // KV tiles per range
    float scale_log2;   // scale * log2(e)
    uint32_t flags;
};

template <int D, int NS>
struct SmemLayout {
    static_assert(D == 64 || D == 128, "head dim 64 or 128");
    static constexpr int NCH = D / CHUNK_ELEMS;
    static constexpr int TILE_BYTES = NCH * CHUNK_BYTES;  // 128 rows x D x 2 bytes
    static constexpr int Q_OFF = 0;                        // two query tiles
    static constexpr int K_OFF = Q_OFF + 2 * TILE_BYTES;
    static constexpr int V_OFF = K_OFF + NS * TILE_BYTES;
    static constexpr int FM_OFF = V_OFF + NS * TILE_BYTES;  // final max  float [2][128]
    static constexpr int FL_OFF = FM_OFF + 2 * BM * 4;      // final sum  float [2][128]
    static constexpr int BAR_OFF = FL_OFF + 2 * BM * 4;
    // q_full[2], k_full[NS], k_empty[NS], v_full[NS], v_empty[NS], s_full[2],
    // p_full[2], o_final[2], stats[2], o_free[2], q_empty[2], drain
    static constexpr int NBAR = 2 + 4 * NS + 2 * 6 + 1;
    static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;  // tmem base, error flag
    static constexpr int BYTES = MISC_OFF + 16;
    static constexpr int ALLOC = BYTES + 1024;  // slack to align the base to 1024
    // The CTA takes all 512 TMEM columns, so no second CTA may share its SM: the
    // shared-memory request alone must rule that out.
    static_assert(2 * ALLOC > 232448, "one CTA per SM must be guaranteed");
    static_assert(ALLOC <= 232448, "shared memory budget exceeded");
};

__device__ int g_attn_status;  // first error code a kernel recorded (0 = none)

struct Ctx {
    volatile int* err;  // per-CTA error flag in shared memory
};

__device__ __forceinline__ void raise_error(const Ctx& c, int code) {
    *c.err = 1;
    atomicCAS(&g_attn_status, 0, code);
}

// Bounded wait for the completion of the phase with `parity`.  Gives up when the CTA
// error flag is set or after WAIT_LIMIT_NS.
__device__ __forceinline__ bool wait_bounded(const Ctx& c, uint32_t bar, uint32_t parity) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    while (true) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if (*c.err) return false;
        if (ptx::globaltimer_ns() - t0 > WAIT_LIMIT_NS) {
            raise_error(c, STATUS_TIMEOUT);
            return false;
        }
    }
}

// Used on the way out: ignores the error flag, bounded by DRAIN_LIMIT_NS.
__device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = ptx::globaltimer_ns();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (ptx::globaltimer_ns() - t0 > DRAIN_LIMIT_NS) return false;
    }
    return true;
}

// Every lane waits, then the warp agrees: one lane's failure fails the warp, so
// warp-collective tcgen05 instructions that follow are never divergent.
__device__ __forceinline__ bool warp_wait(const Ctx& c, uint32_t bar, uint32_t parity) {
    const bool ok = wait_bounded(c, bar, parity);
    return __all_sync(0xffffffffu, ok);
}

template <bool IS_BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    if constexpr (IS_BF16) return ptx::pack_bf16x2(lo, hi);
    else return ptx::pack_f16x2(lo, hi);
}

// One work unit: query pair qp (rows qp*256 .. +255) of head bh, over the KV tiles
// [kv0, kv0 + n[t]) for query tile t (0 tiles when the query tile lies past Sq or,
// causally, before the range).  Units are numbered so that causal grids go heaviest
// first (the last query pairs of every head first) and non-causal grids keep a head's
// query pairs adjacent (concurrent units share its K/V in L2); the KV ranges of one
// (query pair, head) are adjacent.
struct Unit {
    int qp, bh, split, kv0;
    int n[2];
};

// Causal visibility bound of packed rows first..last: the last key visible to the
// row at the largest query position (LEAST = false) or to the row at the smallest one
// (LEAST = true).  The rows span a head boundary only with grouped heads.
template <bool LEAST>
__device__ __forceinline__ int tile_vis(int first, int last, const Params& p) {
    int pos;
    if (p.sq_head == p.Sq) {
        pos = LEAST ? first : last;
    } else if (first / p.sq_head != last / p.sq_head) {
        pos = LEAST ? 0 : p.sq_head - 1;
    } else {
        pos = (LEAST ? first : last) % p.sq_head;
    }
    return pos + p.causal_off;
}

template <bool CAUSAL, bool SPLIT, bool GEN>
__device__ __forceinline__ Unit decode_unit(int u, const Params& p) {
    Unit w;
    w.split = SPLIT ? u % p.n_splits : 0;
    const int rest = SPLIT ? u / p.n_splits : u;
    if constexpr (CAUSAL) {
        w.qp = p.n_qp - 1 - rest / p.BH;
        w.bh = rest % p.BH;
    } else {
        w.qp = rest % p.n_qp;
        w.bh = rest / p.n_qp;
    }
    const int n_all = (p.Sk + BN - 1) / BN;
    w.kv0 = SPLIT ? w.split * p.chunk_tiles : 0;
    const int kv_end = SPLIT ? min(n_all, w.kv0 + p.chunk_tiles) : n_all;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const int first = w.qp * ROWS_PER_CTA + BM * t;
        int end = kv_end;
        if (CAUSAL) {
            // the last key any row of the tile sees
            const int last = min(first + BM - 1, p.Sq - 1);
            const int vis = GEN ? tile_vis<false>(first, last, p) : last;
            end = vis < 0 ? 0 : min(end, vis / BN + 1);
        }
        w.n[t] = (first >= p.Sq) ? 0 : max(0, end - w.kv0);
    }
    return w;
}

// --------------------------------------------------------------------------- softmax
// Row max of 64 scores, folded into eight running accumulators.
__device__ __forceinline__ void max64(const uint32_t* s, float (&a)[8]) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
#pragma unroll
        for (int k = 0; k < 8; k += 2)
            a[i] = ptx::max3(a[i], __uint_as_float(s[i + 8 * k]), __uint_as_float(s[i + 8 * k + 8]));
    }
}

// With a negative scale the scores are negated as they are read (scale * s =
// |scale| * (-s)), so the softmax below always takes a max and multiplies by |scale|.
template <bool NEG>
__device__ __forceinline__ void load_scores(uint32_t tS, uint32_t (&s)[128], int half) {
    ptx::tmem_ld32(tS + 64 * half, *reinterpret_cast<uint32_t(*)[32]>(&s[64 * half]));
    ptx::tmem_ld32(tS + 64 * half + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[64 * half + 32]));
}
template <bool NEG>
__device__ __forceinline__ void scores_ready(uint32_t (&s)[128], int half) {
    ptx::reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&s[64 * half]));
    ptx::reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&s[64 * half + 32]));
    if constexpr (NEG) {
#pragma unroll
        for (int k = 0; k < 64; ++k) s[64 * half + k] ^= 0x80000000u;
    }
}

// p = 2^(s * c - m) for 32 column pairs starting at pair k0, packed to 16 bits into
// pk, the row sum accumulated in the packed pair acc.
template <bool IS_BF16>
__device__ __forceinline__ void exp_pairs32(const uint32_t (&s)[128], int k0, float c,
                                            float neg_m, uint32_t (&pk)[64], uint64_t& acc) {
    const uint64_t c2 = ptx::f32x2(c, c), m2 = ptx::f32x2(neg_m, neg_m);
#pragma unroll
    for (int k = k0; k < k0 + 32; ++k) {
        float x0, x1;
        ptx::f32x2_split(
            ptx::fma2(ptx::f32x2(__uint_as_float(s[2 * k]), __uint_as_float(s[2 * k + 1])), c2, m2),
            x0, x1);
        const float p0 = ptx::ex2(x0), p1 = ptx::ex2(x1);
        acc = ptx::add2(acc, ptx::f32x2(p0, p1));
        pk[k] = pack2<IS_BF16>(p0, p1);
    }
}

__device__ __forceinline__ float sum_pair(uint64_t acc) {
    float a0, a1;
    ptx::f32x2_split(acc, a0, a1);
    return a0 + a1;
}

// One KV tile of the query row this thread owns, with the masking decided at compile
// time (MASK: keys past tile-relative index `lim` are invisible): read S_j from TMEM,
// update the running max (lazily), exponentiate, accumulate the normaliser and write
// P_j (16-bit) over S_j.  The exponentials run on the SFU (ex2.approx); the
// scale-and-shift and the row sum use packed f32x2 arithmetic, two columns per
// instruction.  c = |scale| * log2(e) > 0 (the host passes 1e-30 for a zero scale:
// every visible p is then 2^(~1e-28) = 1.0f exactly, the uniform weights a zero
// scale gives, and masked scores stay -inf).  Returns alpha, the factor O must be
// scaled by before P_j V_j is added (1 = none).
template <bool IS_BF16, bool NEG, bool MASK, bool GEN>
__device__ __forceinline__ float softmax_tile_body(uint32_t tS, int j, int lim, float c,
                                                   float& m_used, float& l) {
    uint32_t s[128];
    load_scores<NEG>(tS, s, 0);
    ptx::tmem_wait_ld();
    scores_ready<NEG>(s, 0);
    // the second half's load runs under the first half's reduction
    load_scores<NEG>(tS, s, 1);
    float a[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = -INFINITY;
    if constexpr (MASK) {
        ptx::tmem_wait_ld();
        scores_ready<NEG>(s, 1);
#pragma unroll
        for (int k = 0; k < 128; ++k)
            if (k > lim) s[k] = __float_as_uint(-INFINITY);
        max64(&s[0], a);
    } else {
        max64(&s[0], a);
        ptx::tmem_wait_ld();
        scores_ready<NEG>(s, 1);
    }
    max64(&s[64], a);
    const float mx =
        ptx::max3(ptx::max3(a[0], a[1], a[2]), ptx::max3(a[3], a[4], a[5]), fmaxf(a[6], a[7]));
    // mx = -inf only for a row that sees no key of this (masked) tile
    const float m_tile = mx * c;
    float alpha = 1.f;
    if (j == 0) {
        m_used = m_tile;
    } else if (m_tile > m_used + LAZY_RESCALE_LOG2) {
        alpha = ptx::ex2(m_used - m_tile);
        m_used = m_tile;
    }
    // a row that has seen no key yet keeps m = -inf (possible only in a masked tile of
    // the general causal forms: bottom-right offsets, grouped heads); its p must be 0
    const float neg_m = (MASK && GEN && m_used == -INFINITY) ? 0.f : -m_used;

    // p = 2^(s * c - m): scale and shift in one packed fma per column pair; the row
    // sums accumulate in packed pairs too (masked scores are -inf and c > 0, so their p
    // is exactly 0)
    uint64_t acc = ptx::f32x2(0.f, 0.f);
    uint32_t pk[64];
    exp_pairs32<IS_BF16>(s, 0, c, neg_m, pk, acc);
    exp_pairs32<IS_BF16>(s, 32, c, neg_m, pk, acc);
    l = l * alpha + sum_pair(acc);
    ptx::tmem_st32(tS, *reinterpret_cast<const uint32_t(*)[32]>(&pk[0]));
    ptx::tmem_st32(tS + 32, *reinterpret_cast<const uint32_t(*)[32]>(&pk[32]));
    return alpha;
}


// An unmasked KV tile after the first of a row's range, without a row-max pass in the
// common case: the running max the row already has (m_used, finite) is used directly,
// p = 2^(s c - m_used), and the tile's row max is only taken when the row sum exceeds
// 2^LIMIT_LOG2, which every tile whose max stays within LIMIT_LOG2 - 7 of the kept
// one passes (128 values of at most 2^(LIMIT_LOG2 - 7)).  A warp with a row above the
// limit (rare once the first tiles have set the max) reloads its scores from tensor
// memory (P is not written yet), takes the row max, moves the kept max to it when it
// is higher (so the dominant p is then exactly 1) and recomputes; rows of the warp
// whose max did not move recompute the same values.  O and l stay relative to the same
// kept max, so O / l is unchanged, and every kept p is at most 2^LIMIT_LOG2.
// LIMIT_LOG2 = 15 keeps every p inside fp16; 8 matches the lazy threshold of the
// row-max path, so a jump in the max by more than 2^8 always leaves the dominant p
// exactly 1 (one-hot rows then lose nothing to the rounding of their dominant p).
// Returns alpha, as softmax_tile_body does.
template <bool IS_BF16, bool NEG, int LIMIT_LOG2>
__device__ __forceinline__ float softmax_tile_running(uint32_t tS, float c, float& m_used,
                                                      float& l) {
    constexpr float LIMIT = static_cast<float>(1 << LIMIT_LOG2);
    uint32_t s[128];
    uint32_t pk[64];
    uint64_t acc = ptx::f32x2(0.f, 0.f);
    // both halves in one wait: a split load whose second half ran under the first
    // half's exponentials still waited ~160 clocks for it (measured)
    load_scores<NEG>(tS, s, 0);
    load_scores<NEG>(tS, s, 1);
    ptx::tmem_wait_ld();
    scores_ready<NEG>(s, 0);
    scores_ready<NEG>(s, 1);
    exp_pairs32<IS_BF16>(s, 0, c, -m_used, pk, acc);
    exp_pairs32<IS_BF16>(s, 32, c, -m_used, pk, acc);
    float alpha = 1.f;
    if (__any_sync(0xffffffffu, sum_pair(acc) > LIMIT)) {
        load_scores<NEG>(tS, s, 0);
        load_scores<NEG>(tS, s, 1);
        ptx::tmem_wait_ld();
        scores_ready<NEG>(s, 0);
        scores_ready<NEG>(s, 1);
        float a[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) a[i] = -INFINITY;
        max64(&s[0], a);
        max64(&s[64], a);
        const float mx = ptx::max3(ptx::max3(a[0], a[1], a[2]), ptx::max3(a[3], a[4], a[5]),
                                   fmaxf(a[6], a[7]));
        const float m_tile = mx * c;
        if (m_tile > m_used) {
            alpha = ptx::ex2(m_used - m_tile);
            m_used = m_tile;
        }
        acc = ptx::f32x2(0.f, 0.f);
        exp_pairs32<IS_BF16>(s, 0, c, -m_used, pk, acc);
        exp_pairs32<IS_BF16>(s, 32, c, -m_used, pk, acc);
    }
    l = l * alpha + sum_pair(acc);
    ptx::tmem_st32(tS, *reinterpret_cast<const uint32_t(*)[32]>(&pk[0]));
    ptx::tmem_st32(tS + 32, *reinterpret_cast<const uint32_t(*)[32]>(&pk[32]));
    return alpha;
}

// LIMIT_LOG2: see softmax_tile_running.
template <bool IS_BF16, bool CAUSAL, bool NEG, bool GEN, int LIMIT_LOG2>
__device__ __forceinline__ float softmax_tile(uint32_t tS, int j, int kv0, int Sk, int row_vis,
                                              int tile_vis_min, float c, float& m_used,
                                              float& l) {
    const bool need_mask = (kv0 + BN > Sk) || (CAUSAL && kv0 + BN - 1 > tile_vis_min);
    if (need_mask) {
        int lim = Sk - 1 - kv0;
        if (CAUSAL) lim = min(lim, row_vis - kv0);
        return softmax_tile_body<IS_BF16, NEG, true, GEN>(tS, j, lim, c, m_used, l);
    }
    if (j > 0) return softmax_tile_running<IS_BF16, NEG, LIMIT_LOG2>(tS, c, m_used, l);
    return softmax_tile_body<IS_BF16, NEG, false, GEN>(tS, j, 0, c, m_used, l);
}

// O = 0, LSE = -inf for a row that sees no key (whole pass: 16-bit O; split pass: the
// fp32 partials of the range).
template <int D, bool SPLIT>
__device__ __forceinline__ void write_empty_row(const Params& p, int64_t head_row, int bh,
                                                int qrow) {
    if constexpr (SPLIT) {
        float4* dst = reinterpret_cast<float4*>(p.ws_o + (head_row * p.Sq + qrow) * p.d_out);
#pragma unroll 1
        for (int c = 0; c < p.d_out / 4; ++c) dst[c] = make_float4(0.f, 0.f, 0.f, 0.f);
        p.ws_lse[head_row * p.Sq + qrow] = -INFINITY;
    } else {
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.o) +
                                              (static_cast<int64_t>(bh) * p.Sq + qrow) * p.d_out);
#pragma unroll 1
        for (int c = 0; c < p.d_out / 8; ++c) dst[c] = make_uint4(0u, 0u, 0u, 0u);
        if (p.lse != nullptr) p.lse[static_cast<int64_t>(bh) * p.Sq + qrow] = -INFINITY;
    }
}

// 8 normalised output values (columns 8c .. 8c+7) of one row: fp32 partials (split
// pass) or one rounding to 16 bits.
template <int D, bool IS_BF16, bool SPLIT>
__device__ __forceinline__ void store_o8(const Params& p, int64_t head_row, int bh, int qrow,
                                         int c, const float (&f)[8]) {
    if constexpr (SPLIT) {
        float4* dst = reinterpret_cast<float4*>(p.ws_o + (head_row * p.Sq + qrow) * p.d_out + 8 * c);
        dst[0] = make_float4(f[0], f[1], f[2], f[3]);
        dst[1] = make_float4(f[4], f[5], f[6], f[7]);
    } else {
        uint16_t* o = reinterpret_cast<uint16_t*>(p.o) + (static_cast<int64_t>(bh) * p.Sq + qrow) * p.d_out;
        *reinterpret_cast<uint4*>(o + 8 * c) =
            make_uint4(pack2<IS_BF16>(f[0], f[1]), pack2<IS_BF16>(f[2], f[3]),
                       pack2<IS_BF16>(f[4], f[5]), pack2<IS_BF16>(f[6], f[7]));
    }
}

// The r-th unit of this CTA in a boustrophedon order over the grid (round r takes
// units r*G .. r*G+G-1, in reverse CTA order on odd rounds), so with heaviest-first
// units every CTA's total stays close to the others'.  -1 when none is left.
__device__ __forceinline__ int unit_of(int r, int n_units) {
    const int G = static_cast<int>(gridDim.x);
    const int b = static_cast<int>(blockIdx.x);
    const int u = r * G + ((r & 1) ? G - 1 - b : b);
    return u < n_units ? u : -1;
}

// GEN (causal only): the general causal forms -- a nonzero offset (bottom-right
// alignment) or grouped query heads packed into one sequence; without it a row's
// position is its row index and the offset is 0, and no row is ever fully masked.
// DEC (decode shapes: every unit's rows fit in query tile 0, so tile 1 would be empty):
// both softmax warpgroups work on tile 0's rows, warpgroup t on the unit's KV tiles
// t, t + 2, t + 4, ... with its own running max, sum and O_t accumulator; the epilogue
// merges the two halves exactly (like a split in two).  Two softmax chains then share
// each KV tile stream, and only Q tile 0 is loaded.
template <int D, int NS, bool IS_BF16, bool CAUSAL, bool NEG, bool SPLIT, bool GEN, bool DEC>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const Params p) {
    using L = SmemLayout<D, NS>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = ptx::smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
    const uint32_t sbase = ptx::smem_u32(smem);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const uint32_t sQ = sbase + L::Q_OFF;
    const uint32_t sK = sbase + L::K_OFF;
    const uint32_t sV = sbase + L::V_OFF;
    float* s_fm = reinterpret_cast<float*>(smem + L::FM_OFF);
    float* s_fl = reinterpret_cast<float*>(smem + L::FL_OFF);
    const uint32_t bars = sbase + L::BAR_OFF;
    auto B_QF = [&](int t) { return bars + 8u * t; };                  // Q_t loaded
    auto B_KF = [&](int s) { return bars + 8u * (2 + s); };
    auto B_KE = [&](int s) { return bars + 8u * (2 + NS + s); };
    auto B_VF = [&](int s) { return bars + 8u * (2 + 2 * NS + s); };
    auto B_VE = [&](int s) { return bars + 8u * (2 + 3 * NS + s); };
    auto B_SF = [&](int t) { return bars + 8u * (2 + 4 * NS + t); };   // S_t,j in TMEM
    auto B_PF = [&](int t) { return bars + 8u * (4 + 4 * NS + t); };   // P_t,j (+ O_t) ready
    auto B_OF = [&](int t) { return bars + 8u * (6 + 4 * NS + t); };   // last PV_t done
    auto B_ST = [&](int t) { return bars + 8u * (8 + 4 * NS + t); };   // final m, l in smem
    auto B_OE = [&](int t) { return bars + 8u * (10 + 4 * NS + t); };  // O_t, m, l read out
    auto B_QE = [&](int t) { return bars + 8u * (12 + 4 * NS + t); };  // Q_t free
    const uint32_t B_DR = bars + 8u * (14 + 4 * NS);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
    Ctx ctx{reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4)};
    const int n_units = p.n_qp * p.BH * p.n_splits;

    // ---- set-up (once per CTA)
    if (threadIdx.x == 0) {
        for (int t = 0; t < 2; ++t) {
            ptx::mbar_init(B_QF(t), 1);
            ptx::mbar_init(B_SF(t), 1);
            ptx::mbar_init(B_PF(t), 4);  // one arrival per softmax warp
            ptx::mbar_init(B_OF(t), 1);
            ptx::mbar_init(B_ST(t), 4);  // one arrival per softmax warp
            ptx::mbar_init(B_OE(t), 4);  // one arrival per epilogue warp
        }
        for (int s = 0; s < NS; ++s) {
            ptx::mbar_init(B_KF(s), 1);
            ptx::mbar_init(B_KE(s), 1);
            ptx::mbar_init(B_VF(s), 1);
            ptx::mbar_init(B_VE(s), 1);
        }
        ptx::mbar_init(B_QE(0), 1);
        ptx::mbar_init(B_QE(1), 1);
        ptx::mbar_init(B_DR, 1);
        *ctx.err = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 13 && lane == 0) {
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_k);
        ptx::prefetch_tmap(&tm_v);
    }
    if (warp == 14) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // Barrier phases run on across units: every role visits the same units in the same
    // order and counts (a) KV tiles per query tile for S / P, (b) KV tiles of the unit
    // for the K / V ring, (c) units with rows in query tile t for the per-unit
    // hand-offs (Q, final O, statistics, O read-out).

    if (warp < 8) {
        // ================================================================ softmax
        ptx::setmaxnreg_inc<200>();
        const int t = warp >> 2;                    // query tile
        const int wq = warp & 3;                    // TMEM lane quarter
        const int row = wq * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t tS = tmem + lane_base + TMEM_S + 128u * t;
        const uint32_t tO = tmem + lane_base + TMEM_O + D * t;
        const float c_abs = fabsf(p.scale_log2);
        bool ok = true;
        uint32_t it = 0;  // KV tiles of this query tile so far (S / P phases)
        uint32_t ut = 0;  // units with rows in this query tile so far
        for (int r = 0; ok; ++r) {
            const int u = unit_of(r, n_units);
            if (u < 0) break;
            const Unit w = decode_unit<CAUSAL, SPLIT, GEN>(u, p);
            const int q0t = w.qp * ROWS_PER_CTA + (DEC ? 0 : BM * t);
            const int qrow = q0t + row;
            // DEC: warpgroup t takes the unit's KV tiles t, t + 2, ...
            const int n_t = DEC ? (w.n[0] + 1 - t) >> 1 : w.n[t];
            int row_vis = qrow, tile_vis_min = q0t;
            if (GEN && n_t > 0) {
                row_vis = (p.sq_head == p.Sq ? qrow : qrow % p.sq_head) + p.causal_off;
                tile_vis_min = tile_vis<true>(q0t, min(q0t + BM - 1, p.Sq - 1), p);
            }
            float m_used = -INFINITY;
            float l = 0.f;
            for (int j = 0; j < n_t; ++j, ++it) {
                if (!(ok = warp_wait(ctx, B_SF(t), it & 1))) break;
                ptx::tc_fence_after();
                const int kt = DEC ? 2 * j + t : j;  // the KV tile within the unit's range
                const float alpha = softmax_tile<IS_BF16, CAUSAL, NEG, GEN, 15>(
                    tS, j, (w.kv0 + kt) * BN, p.Sk, row_vis, tile_vis_min, c_abs, m_used, l);
                // O_t holds the sum over tiles < j (PV_t,j-1 completed before S_t,j);
                // bring it to the new max before PV_t,j adds to it
                if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t ov[32];
                        ptx::tmem_ld32(tO + 32 * c, ov);
                        ptx::tmem_wait_ld();
                        ptx::reg_fence32(ov);
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
                        ptx::tmem_st32(tO + 32 * c, ov);
                    }
                }
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(B_PF(t));
            }
            if (!ok || n_t == 0) continue;
            // the epilogue must be done with the previous unit's statistics
            if (!(ok = warp_wait(ctx, B_OE(t), (ut & 1) ^ 1))) break;
            s_fm[t * BM + row] = m_used;
            s_fl[t * BM + row] = l;
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(B_ST(t));
            ++ut;
        }
    } else if (warp < 12) {
        // ================================================================ epilogue
        ptx::setmaxnreg_dec<48>();
        const int wq = warp & 3;
        const int row = wq * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
        bool ok = true;
        uint32_t ut[2] = {0, 0};
        for (int r = 0; ok; ++r) {
            const int u = unit_of(r, n_units);
            if (u < 0) break;
            const Unit w = decode_unit<CAUSAL, SPLIT, GEN>(u, p);
            const int64_t head_row = static_cast<int64_t>(w.split) * p.BH + w.bh;
            if constexpr (DEC) {
                // tile 0's rows from two halves: O_t, m_t, l_t over KV tiles t, t + 2, ...
                const int qrow = w.qp * ROWS_PER_CTA + row;
                const bool store = qrow < p.Sq;
                const int nt1 = w.n[0] >> 1;
                if (w.n[0] == 0) {
                    if (store) write_empty_row<D, SPLIT>(p, head_row, w.bh, qrow);
                    continue;
                }
                if (!(ok = warp_wait(ctx, B_ST(0), ut[0] & 1))) break;
                if (!(ok = warp_wait(ctx, B_OF(0), ut[0] & 1))) break;
                if (nt1 > 0) {
                    if (!(ok = warp_wait(ctx, B_ST(1), ut[1] & 1))) break;
                    if (!(ok = warp_wait(ctx, B_OF(1), ut[1] & 1))) break;
                }
                ptx::tc_fence_after();
                const float m0 = s_fm[row], l0 = s_fl[row];
                const float m1 = nt1 > 0 ? s_fm[BM + row] : -INFINITY;
                const float l1 = nt1 > 0 ? s_fl[BM + row] : 0.f;
                const float mx = fmaxf(m0, m1);
                // weights of the halves (0 for a half that saw no key)
                const float a0 = m0 == -INFINITY ? 0.f : ptx::ex2(m0 - mx);
                const float a1 = m1 == -INFINITY ? 0.f : ptx::ex2(m1 - mx);
                const float lt = l0 * a0 + l1 * a1;
                const float inv = lt > 0.f ? 1.f / lt : 0.f;
                const float w0 = a0 * inv, w1 = a1 * inv;
                const float lse_row =
                    lt > 0.f ? (mx + log2f(lt)) * 0.69314718055994530942f : -INFINITY;
                const uint32_t tO0 = tmem + lane_base + TMEM_O;
#pragma unroll 1
                for (int c = 0; c < p.d_out / 8; ++c) {
                    uint32_t o0[8], o1[8];
                    ptx::tmem_ld8(tO0 + 8 * c, o0);
                    if (nt1 > 0) ptx::tmem_ld8(tO0 + D + 8 * c, o1);
                    ptx::tmem_wait_ld();
                    ptx::reg_fence8(o0);
                    if (nt1 > 0) ptx::reg_fence8(o1);
                    float f[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        f[e] = __uint_as_float(o0[e]) * w0 +
                               (nt1 > 0 ? __uint_as_float(o1[e]) * w1 : 0.f);
                    if (store) store_o8<D, IS_BF16, SPLIT>(p, head_row, w.bh, qrow, c, f);
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    ptx::mbar_arrive(B_OE(0));
                    if (nt1 > 0) ptx::mbar_arrive(B_OE(1));
                }
                ++ut[0];
                if (nt1 > 0) ++ut[1];
                if (store) {
                    if constexpr (SPLIT)
                        p.ws_lse[head_row * p.Sq + qrow] = lse_row;
                    else if (p.lse != nullptr)
                        p.lse[static_cast<int64_t>(w.bh) * p.Sq + qrow] = lse_row;
                }
                continue;
            }
            if constexpr (!DEC) for (int t = 0; ok && t < 2; ++t) {
                const int qrow = w.qp * ROWS_PER_CTA + BM * t + row;
                const bool store = qrow < p.Sq;
                if (w.n[t] == 0) {
                    // no key of the unit's range is visible to these rows: O = 0 and
                    // LSE = -inf (the empty sum)
                    if (store) write_empty_row<D, SPLIT>(p, head_row, w.bh, qrow);
                    continue;
                }
                if (!(ok = warp_wait(ctx, B_ST(t), ut[t] & 1))) break;
                if (!(ok = warp_wait(ctx, B_OF(t), ut[t] & 1))) break;
                ptx::tc_fence_after();
                const float m_used = s_fm[t * BM + row];
                const float l = s_fl[t * BM + row];
                // l = 0 only for a row with no visible key in a split range
                const float inv_l = l > 0.f ? 1.f / l : 0.f;
                const float lse_row =
                    l > 0.f ? (m_used + log2f(l)) * 0.69314718055994530942f : -INFINITY;
                const uint32_t tO = tmem + lane_base + TMEM_O + D * t;
                if constexpr (SPLIT) {
                    // partial O / l and LSE of this KV range, fp32
                    float* orow = p.ws_o + (head_row * p.Sq + qrow) * p.d_out;
#pragma unroll 1
                    for (int c = 0; c < p.d_out / 16; ++c) {
                        uint32_t ov[16];
                        ptx::tmem_ld16(tO + 16 * c, ov);
                        ptx::tmem_wait_ld();
                        ptx::reg_fence16(ov);
                        if (store) {
                            float4* dst = reinterpret_cast<float4*>(orow + 16 * c);
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                dst[e] = make_float4(__uint_as_float(ov[4 * e]) * inv_l,
                                                     __uint_as_float(ov[4 * e + 1]) * inv_l,
                                                     __uint_as_float(ov[4 * e + 2]) * inv_l,
                                                     __uint_as_float(ov[4 * e + 3]) * inv_l);
                        }
                    }
                } else {
                    // O / l in fp32, one rounding to 16 bits; LSE in natural log
                    uint16_t* orow = reinterpret_cast<uint16_t*>(p.o) +
                                     (static_cast<int64_t>(w.bh) * p.Sq + qrow) * p.d_out;
#pragma unroll 1
                    for (int c = 0; c < p.d_out / 16; ++c) {
                        uint32_t ov[16];
                        ptx::tmem_ld16(tO + 16 * c, ov);
                        ptx::tmem_wait_ld();
                        ptx::reg_fence16(ov);
                        uint32_t packed[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            packed[e] = pack2<IS_BF16>(__uint_as_float(ov[2 * e]) * inv_l,
                                                       __uint_as_float(ov[2 * e + 1]) * inv_l);
                        if (store) {
                            uint4* dst = reinterpret_cast<uint4*>(orow + 16 * c);
                            dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                            dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
                        }
                    }
                }
                // O_t and the statistics are read: the next unit may overwrite them
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(B_OE(t));
                ++ut[t];
                if (store) {
                    if constexpr (SPLIT)
                        p.ws_lse[head_row * p.Sq + qrow] = lse_row;
                    else if (p.lse != nullptr)
                        p.lse[static_cast<int64_t>(w.bh) * p.Sq + qrow] = lse_row;
                }
            }
        }
    } else {
        ptx::setmaxnreg_dec<64>();
        if (warp == 12) {
            // ============================================================ MMA issuer
            if (lane == 0) {
                constexpr uint32_t fmt = IS_BF16 ? 1u : 0u;
                constexpr uint32_t idesc_qk = ptx::idesc_f16(fmt, BM, BN, 0);
                constexpr uint32_t idesc_pv = ptx::idesc_f16(fmt, BM, D, 1);
                // Descriptors: the high word is common to every operand tile; per MMA only
                // the start-address field of the low word moves, by a compile-time offset.
                constexpr uint32_t desc_hi = ptx::smem_desc_hi_sw128(1024);
                const uint32_t dq0 = ptx::smem_desc_lo(sQ, 16);
                const uint32_t dk0 = ptx::smem_desc_lo(sK, 16);
                const uint32_t dv0 = ptx::smem_desc_lo(sV, CHUNK_BYTES);
                constexpr uint32_t TILE16 = L::TILE_BYTES >> 4;
                // S_t = Q_t K^T for the K tile in ring slot `slot`
                auto issue_s = [&](int t, int slot) {
                    // (DEC: both S accumulators take query tile 0)
                    const uint32_t qd = dq0 + static_cast<uint32_t>(DEC ? 0 : t) * TILE16;
                    const uint32_t kd = dk0 + static_cast<uint32_t>(slot) * TILE16;
                    const uint32_t d_tmem = tmem + TMEM_S + 128u * t;
                    // K-steps of 16: +32 bytes inside a 128-byte row, +16 KB per 64 columns
                    ptx::mma_ss_off<0, 0>(d_tmem, qd, kd, desc_hi, idesc_qk, 0u);
                    ptx::mma_ss_off<2, 2>(d_tmem, qd, kd, desc_hi, idesc_qk, 1u);
                    ptx::mma_ss_off<4, 4>(d_tmem, qd, kd, desc_hi, idesc_qk, 1u);
                    ptx::mma_ss_off<6, 6>(d_tmem, qd, kd, desc_hi, idesc_qk, 1u);
                    if constexpr (D == 128) {
                        constexpr uint32_t C16 = CHUNK_BYTES >> 4;
                        ptx::mma_ss_off<C16, C16>(d_tmem, qd, kd, desc_hi, idesc_qk, 1u);
                        ptx::mma_ss_off<C16 + 2, C16 + 2>(d_tmem, qd, kd, desc_hi, idesc_qk, 1u);
                        ptx::mma_ss_off<C16 + 4, C16 + 4>(d_tmem, qd, kd, desc_hi, idesc_qk, 1u);
                        ptx::mma_ss_off<C16 + 6, C16 + 6>(d_tmem, qd, kd, desc_hi, idesc_qk, 1u);
                    }
                    ptx::mma_commit(B_SF(t));
                };
                // O_t (+)= P_t V for the V tile in ring slot `slot`
                auto issue_pv = [&](int t, int slot, bool first) {
                    const uint32_t vd = dv0 + static_cast<uint32_t>(slot) * TILE16;
                    const uint32_t a_tmem = tmem + TMEM_S + 128u * t;
                    const uint32_t d_tmem = tmem + TMEM_O + D * t;
                    // K-steps of 16 keys: 8 TMEM columns of P, 2 KB of V
                    ptx::mma_ts_off<0, 0>(d_tmem, a_tmem, vd, desc_hi, idesc_pv, first ? 0u : 1u);
                    ptx::mma_ts_off<8, 128>(d_tmem, a_tmem, vd, desc_hi, idesc_pv, 1u);
                    ptx::mma_ts_off<16, 256>(d_tmem, a_tmem, vd, desc_hi, idesc_pv, 1u);
                    ptx::mma_ts_off<24, 384>(d_tmem, a_tmem, vd, desc_hi, idesc_pv, 1u);
                    ptx::mma_ts_off<32, 512>(d_tmem, a_tmem, vd, desc_hi, idesc_pv, 1u);
                    ptx::mma_ts_off<40, 640>(d_tmem, a_tmem, vd, desc_hi, idesc_pv, 1u);
                    ptx::mma_ts_off<48, 768>(d_tmem, a_tmem, vd, desc_hi, idesc_pv, 1u);
                    ptx::mma_ts_off<56, 896>(d_tmem, a_tmem, vd, desc_hi, idesc_pv, 1u);
                };
                bool ok = true;
                uint32_t kv = 0;          // K/V ring position of the unit's first tile
                uint32_t pit[2] = {0, 0};  // P phases per query tile
                uint32_t ut[2] = {0, 0};   // units with rows per query tile
                uint32_t nu = 0;           // units so far (Q phases)
                // DEC order, KV tile j to accumulator t = j % 2:
                //   S0,0 S1,1 | PV0,0 S0,2 | PV1,1 S1,3 | PV0,2 S0,4 | ...
                // each K / V ring position is used by one product.
                for (int r = 0; DEC && ok; ++r) {
                    const int u = unit_of(r, n_units);
                    if (u < 0) break;
                    const Unit w = decode_unit<CAUSAL, SPLIT, GEN>(u, p);
                    const int n = w.n[0];
                    if (n == 0) continue;  // a range no row of the unit sees
                    const int nt[2] = {(n + 1) >> 1, n >> 1};
                    auto slot = [&](int j) { return static_cast<int>((kv + j) % NS); };
                    auto phase = [&](int j) { return ((kv + j) / NS) & 1u; };
                    if (!(ok = wait_bounded(ctx, B_QF(0), nu & 1))) break;
                    for (int j = 0; ok && j < 2 && j < n; ++j) {
                        if (!(ok = wait_bounded(ctx, B_KF(slot(j)), phase(j)))) break;
                        ptx::tc_fence_after();
                        issue_s(j, slot(j));
                        ptx::mma_commit(B_KE(slot(j)));
                        if (j == n - 1) ptx::mma_commit(B_QE(0));  // the unit's last S is issued
                    }
                    for (int j = 0; ok && j < n; ++j) {
                        const int t = j & 1, i = j >> 1;
                        if (!(ok = wait_bounded(ctx, B_VF(slot(j)), phase(j)))) break;
                        // t is a run-time value here: the counters are picked by selects (an
                        // index by t would put them in local memory, on this thread's path)
                        if (!(ok = wait_bounded(ctx, B_PF(t), (t ? pit[1] : pit[0]) & 1))) break;
                        if (t) ++pit[1];
                        else ++pit[0];
                        // the first P V into O_t overwrites it: the epilogue must have read
                        // the previous unit's O_t
                        if (i == 0 &&
                            !(ok = wait_bounded(ctx, B_OE(t), ((t ? ut[1] : ut[0]) & 1) ^ 1)))
                            break;
                        ptx::tc_fence_after();
                        issue_pv(t, slot(j), i == 0);
                        ptx::mma_commit(B_VE(slot(j)));
                        if (i == (t ? nt[1] : nt[0]) - 1) ptx::mma_commit(B_OF(t));
                        if (j + 2 < n) {
                            if (!(ok = wait_bounded(ctx, B_KF(slot(j + 2)), phase(j + 2)))) break;
                            ptx::tc_fence_after();
                            issue_s(t, slot(j + 2));
                            ptx::mma_commit(B_KE(slot(j + 2)));
                            if (j + 2 == n - 1) ptx::mma_commit(B_QE(0));  // last S issued
                        }
                    }
                    for (int t = 0; t < 2; ++t) ut[t] += nt[t] > 0 ? 1u : 0u;
                    kv += static_cast<uint32_t>(n);
                    ++nu;
                }
                // Tile 0 runs ahead across units: once its last P V of a unit is issued,
                // the next unit's S_0,0 follows at once (its Q_0 and K_0 loaded: tested
                // without blocking, else after tile 1's work of that step), so the two
                // tiles' softmaxes stay half a period apart across the unit boundary and,
                // causally, tile 0 works while tile 1 finishes its extra diagonal tile.
                // Deadlock-free: the producer loads Q_0, K_0, Q_1, V_0, K_1, ... of a
                // unit; Q_0 of the next unit needs only tile 0's last S of this unit
                // (Q_t is freed per tile), and K_0 of the next unit needs the ring slot
                // of K at tile n_max - NS of this unit, whose S MMAs were issued before
                // tile 0's last step when n_0 >= n_max - NS + 1 (the lookahead's
                // condition).
                bool s0_pre = false;  // S_0,0 of the unit about to start is issued
                auto next_unit = [&](int r0, Unit& nx) {
                    for (int r1 = r0 + 1;; ++r1) {
                        const int u1 = unit_of(r1, n_units);
                        if (u1 < 0) return false;
                        nx = decode_unit<CAUSAL, SPLIT, GEN>(u1, p);
                        if (max(nx.n[0], nx.n[1]) > 0) return true;
                    }
                };
                for (int r = 0; !DEC && ok; ++r) {
                    const int u = unit_of(r, n_units);
                    if (u < 0) break;
                    const Unit w = decode_unit<CAUSAL, SPLIT, GEN>(u, p);
                    const int n_t[2] = {w.n[0], w.n[1]};
                    const int n_max = max(n_t[0], n_t[1]);
                    if (n_max == 0) continue;  // a split range no query row of the unit sees
                    auto slot = [&](int j) { return static_cast<int>((kv + j) % NS); };
                    auto phase = [&](int j) { return ((kv + j) / NS) & 1u; };
                    if (!(ok = (s0_pre || wait_bounded(ctx, B_QF(0), nu & 1)) &&
                               wait_bounded(ctx, B_QF(1), nu & 1) &&
                               wait_bounded(ctx, B_KF(slot(0)), phase(0))))
                        break;
                    ptx::tc_fence_after();
                    if (n_t[0] > 0 && !s0_pre) issue_s(0, slot(0));
                    if (n_t[1] > 0) issue_s(1, slot(0));
                    ptx::mma_commit(B_KE(slot(0)));
                    // Q_t is free once the unit's last S_t is issued (or it has none)
                    if (n_t[0] <= 1 && !s0_pre) ptx::mma_commit(B_QE(0));
                    if (n_t[1] <= 1) ptx::mma_commit(B_QE(1));
                    s0_pre = false;
                    Unit nx;
                    const bool ahead = n_t[0] > 0 && n_t[0] >= n_max - NS + 1 &&
                                       next_unit(r, nx) && nx.n[0] > 0;
                    bool pending = false;  // the lookahead waits for its Q_0 / K_0
                    auto issue_ahead = [&]() {
                        ptx::tc_fence_after();
                        issue_s(0, slot(n_max));
                        if (nx.n[0] == 1) ptx::mma_commit(B_QE(0));
                        s0_pre = true;
                    };
                    for (int j = 0; ok && j < n_max; ++j) {
                        const bool nxt = j + 1 < n_max;
                        if (nxt && !(ok = wait_bounded(ctx, B_KF(slot(j + 1)), phase(j + 1))))
                            break;
                        if (!(ok = wait_bounded(ctx, B_VF(slot(j)), phase(j)))) break;
                        for (int t = 0; t < 2; ++t) {
                            if (j >= n_t[t]) continue;
                            if (!(ok = wait_bounded(ctx, B_PF(t), pit[t] & 1))) break;
                            ++pit[t];
                            // the first P V of a unit overwrites O_t: the epilogue must
                            // have read the previous unit's O_t
                            if (j == 0 && !(ok = wait_bounded(ctx, B_OE(t), (ut[t] & 1) ^ 1)))
                                break;
                            ptx::tc_fence_after();
                            issue_pv(t, slot(j), j == 0);
                            if (j == n_t[t] - 1) ptx::mma_commit(B_OF(t));
                            if (j + 1 < n_t[t]) {
                                issue_s(t, slot(j + 1));
                                if (j + 1 == n_t[t] - 1) ptx::mma_commit(B_QE(t));
                            } else if (t == 0 && ahead) {
                                if (ptx::mbar_test_wait(B_QF(0), (nu + 1) & 1) &&
                                    ptx::mbar_test_wait(B_KF(slot(n_max)), phase(n_max)))
                                    issue_ahead();
                                else
                                    pending = true;
                            }
                        }
                        if (!ok) break;
                        if (pending) {
                            if (!(ok = wait_bounded(ctx, B_QF(0), (nu + 1) & 1) &&
                                       wait_bounded(ctx, B_KF(slot(n_max)), phase(n_max))))
                                break;
                            issue_ahead();
                            pending = false;
                        }
                        ptx::mma_commit(B_VE(slot(j)));
                        if (nxt) ptx::mma_commit(B_KE(slot(j + 1)));
                    }
                    for (int t = 0; t < 2; ++t) ut[t] += n_t[t] > 0 ? 1u : 0u;
                    kv += static_cast<uint32_t>(n_max);
                    ++nu;
                }
                // Every MMA issued above completes before the CTA frees tensor memory.
                ptx::mma_commit(B_DR);
                wait_drain(B_DR, 0);
            }
            __syncwarp();
        } else if (warp == 13) {
            // ============================================================ producer
            if (lane == 0) {
                const bool load_q = !(p.flags & FLAG_SKIP_Q_LOAD);
                uint32_t kv = 0, nu = 0;
                int64_t last_k = -1, last_v = -1;  // ring positions of the last K / V issued
                int64_t last_q[2] = {-1, -1};      // unit count at the last Q_t load
                bool ok = true;
                for (int r = 0; ok; ++r) {
                    const int u = unit_of(r, n_units);
                    if (u < 0) break;
                    const Unit w = decode_unit<CAUSAL, SPLIT, GEN>(u, p);
                    const int q0 = w.qp * ROWS_PER_CTA;
                    const int bh = w.bh;
                    const int n_max = max(w.n[0], w.n[1]);
                    if (n_max == 0) continue;  // nothing to load (the MMA skips it too)
                    // Q_t is free once the previous unit's S_t MMAs completed.  Order of
                    // the loads: Q_0, K_0, Q_1, V_0, K_1, V_1, ... (DEC: only Q_0 is used)
                    auto load_q_tile = [&](int t) {
                        if (!(ok = wait_bounded(ctx, B_QE(t), (nu & 1) ^ 1))) return;
                        if (!load_q) return;
                        ptx::mbar_arrive_expect_tx(B_QF(t), L::TILE_BYTES);
                        for (int c = 0; c < L::NCH; ++c)
                            ptx::tma_load_3d(sQ + t * L::TILE_BYTES + c * CHUNK_BYTES, &tm_q,
                                             B_QF(t), c * CHUNK_ELEMS, q0 + BM * t, bh);
                        last_q[t] = nu;
                    };
                    load_q_tile(0);
                    for (int j = 0; ok && j < n_max; ++j) {
                        const uint32_t pos = kv + j;
                        const int s = static_cast<int>(pos % NS);
                        const uint32_t ph = (pos / NS) & 1;
                        if (!(ok = wait_bounded(ctx, B_KE(s), ph ^ 1))) break;
                        ptx::mbar_arrive_expect_tx(B_KF(s), L::TILE_BYTES);
                        for (int c = 0; c < L::NCH; ++c)
                            ptx::tma_load_3d(sK + s * L::TILE_BYTES + c * CHUNK_BYTES, &tm_k,
                                             B_KF(s), c * CHUNK_ELEMS, (w.kv0 + j) * BN, bh);
                        last_k = pos;
                        if (!DEC && j == 0) {
                            load_q_tile(1);
                            if (!ok) break;
                        }
                        if (!(ok = wait_bounded(ctx, B_VE(s), ph ^ 1))) break;
                        ptx::mbar_arrive_expect_tx(B_VF(s), L::TILE_BYTES);
                        for (int c = 0; c < L::NCH; ++c)
                            ptx::tma_load_3d(sV + s * L::TILE_BYTES + c * CHUNK_BYTES, &tm_v,
                                             B_VF(s), c * CHUNK_ELEMS, (w.kv0 + j) * BN, bh);
                        last_v = pos;
                    }
                    kv += static_cast<uint32_t>(n_max);
                    ++nu;
                }
                // Let every copy this thread started land before the CTA can exit.
                for (int t = 0; t < 2; ++t)
                    if (last_q[t] >= 0) wait_drain(B_QF(t), static_cast<uint32_t>(last_q[t]) & 1);
                for (int64_t q = (last_k - NS + 1 > 0 ? last_k - NS + 1 : 0); q <= last_k; ++q)
                    wait_drain(B_KF(static_cast<int>(q % NS)), (q / NS) & 1);
                for (int64_t q = (last_v - NS + 1 > 0 ? last_v - NS + 1 : 0); q <= last_v; ++q)
                    wait_drain(B_VF(static_cast<int>(q % NS)), (q / NS) & 1);
            }
            __syncwarp();
        }
    }

    // ---- tear-down: every role is out of its loop; free tensor memory
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 14) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace attn
