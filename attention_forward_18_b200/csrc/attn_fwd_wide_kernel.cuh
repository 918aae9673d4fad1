// attn_fwd_wide_kernel.cuh -- the fused attention forward pass for head dimensions 192
// and 256 on a single CTA, where two 128-row query tiles per CTA no longer fit: their O
// accumulators (2 x D fp32 columns) plus S exceed the 512 tensor-memory columns, and a
// 64 KB query tile leaves shared memory for only one 128-key K/V stage.  The library runs
// it for at most 128 packed query rows per K/V head (decoding); larger problems run on
// CTA pairs (attn_fwd_pair_kernel.cuh), which share every K/V tile between 256 rows.
//
// Tile plan: one 128-row query tile per CTA and KV tiles of 64 keys, so the ring holds
// 2 (D = 256) or 3 (D = 192) K/V stages.  Tensor memory: two 64-column S buffers
// (columns 0 and 64) and the D-column O accumulator (from column 128).  With two S
// buffers the MMA thread computes S_{j+1} while the softmax works on S_j:
//   S_0 S_1 | PV_0 S_2 | PV_1 S_3 | ...    (KV tile j in buffer j % 2)
// so the softmax never waits for the MMA; it waits for P V_{j-1} only when it has to
// rescale O (the running max moved by more than 2^8), through a "P V done" barrier.
//
// That barrier is shared by all KV tiles, so a parity wait on it is only unambiguous
// while the barrier can be at most one phase away from the waited one.  Its phase g
// therefore completes on the commit after P V_g AND one arrival of each softmax warp,
// made at tile g + 1 only after the warp saw phase g - 1 complete: no phase can run
// ahead of the softmax, and none can lag it by two.
//
// Warps: 0-3 softmax (thread = row), 4-7 epilogue, 8 MMA issuer, 9 TMA producer,
// 10 tensor-memory allocator, 11 idle; 384 threads.  Units are (128-row query tile,
// head[, KV range]); the persistent grid walks them in the same boustrophedon order,
// and all waits are bounded as in attn_fwd_kernel.cuh.  Softmax arithmetic (exp2 on the
// SFU, packed scale-and-shift and sums, lazy rescale, masking, negative and zero
// scales, grouped heads, causal offsets, split ranges) is the same as there.
#pragma once

#include "attn_fwd_kernel.cuh"

namespace attn {
namespace wide {

constexpr int WBM = 128;                   // query rows per unit
constexpr int WBN = 64;                    // keys per KV tile
constexpr int Q_CHUNK = 128 * 128;         // 128 rows x 128 bytes
constexpr int KV_CHUNK = 64 * 128;         // 64 rows x 128 bytes
constexpr int NUM_THREADS = 384;
constexpr uint32_t TMEM_O = 128;           // O columns; S buffers at 0 and 64

template <int D, int NS>
struct Layout {
    static_assert(D == 192 || D == 256, "head dim 192 or 256");
    static constexpr int NCH = D / CHUNK_ELEMS;
    static constexpr int Q_BYTES = NCH * Q_CHUNK;
    static constexpr int KV_BYTES = NCH * KV_CHUNK;
    static constexpr int Q_OFF = 0;
    static constexpr int K_OFF = Q_OFF + Q_BYTES;
    static constexpr int V_OFF = K_OFF + NS * KV_BYTES;
    static constexpr int FM_OFF = V_OFF + NS * KV_BYTES;  // final max  float [128]
    static constexpr int FL_OFF = FM_OFF + WBM * 4;       // final sum  float [128]
    static constexpr int BAR_OFF = FL_OFF + WBM * 4;
    // q_full, q_empty, k_full[NS], k_empty[NS], v_full[NS], v_empty[NS], s_full[2],
    // p_full[2], pv_done, o_final, stats, o_free, drain
    static constexpr int NBAR = 2 + 4 * NS + 4 + 5;
    static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
    static constexpr int BYTES = MISC_OFF + 16;
    static constexpr int ALLOC = BYTES + 1024;
    static_assert(2 * ALLOC > 232448, "one CTA per SM must be guaranteed");
    static_assert(ALLOC <= 232448, "shared memory budget exceeded");
};

// Unit u: query tile qt (rows qt*128 ..) of head bh, KV tiles [kv0, kv0 + n) of 64 keys.
struct WUnit {
    int qt, bh, split, kv0, n;
};

template <bool CAUSAL, bool SPLIT, bool GEN>
__device__ __forceinline__ WUnit decode_wunit(int u, const Params& p) {
    WUnit w;
    w.split = SPLIT ? u % p.n_splits : 0;
    const int rest = SPLIT ? u / p.n_splits : u;
    if constexpr (CAUSAL) {  // heaviest first: the last query tiles of every head first
        w.qt = p.n_qp - 1 - rest / p.BH;
        w.bh = rest % p.BH;
    } else {
        w.qt = rest % p.n_qp;
        w.bh = rest / p.n_qp;
    }
    const int n_all = (p.Sk + WBN - 1) / WBN;
    w.kv0 = SPLIT ? w.split * p.chunk_tiles : 0;
    int end = SPLIT ? min(n_all, w.kv0 + p.chunk_tiles) : n_all;
    const int first = w.qt * WBM;
    if (CAUSAL) {
        const int last = min(first + WBM - 1, p.Sq - 1);
        const int vis = GEN ? tile_vis<false>(first, last, p) : last;
        end = vis < 0 ? 0 : min(end, vis / WBN + 1);
    }
    w.n = (first >= p.Sq) ? 0 : max(0, end - w.kv0);
    return w;
}

// One 64-key tile of this thread's row (the 128-key version in attn_fwd_kernel.cuh,
// with half the columns): S from TMEM, masking, lazy max, exponentials, normaliser, P
// (16-bit) written over S.  Returns alpha (1 = no rescale of O needed).
template <bool IS_BF16, bool NEG, bool MASK, bool GEN>
__device__ __forceinline__ float softmax64_body(uint32_t tS, int j, int lim, float c,
                                                float& m_used, float& l) {
    uint32_t s[64];
    ptx::tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
    ptx::tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
    ptx::tmem_wait_ld();
    ptx::reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&s[0]));
    ptx::reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&s[32]));
    if constexpr (NEG) {
#pragma unroll
        for (int k = 0; k < 64; ++k) s[k] ^= 0x80000000u;
    }
    if constexpr (MASK) {
#pragma unroll
        for (int k = 0; k < 64; ++k)
            if (k > lim) s[k] = __float_as_uint(-INFINITY);
    }
    float a[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = -INFINITY;
    max64(&s[0], a);
    const float mx =
        ptx::max3(ptx::max3(a[0], a[1], a[2]), ptx::max3(a[3], a[4], a[5]), fmaxf(a[6], a[7]));
    const float m_tile = mx * c;
    float alpha = 1.f;
    if (j == 0) {
        m_used = m_tile;
    } else if (m_tile > m_used + LAZY_RESCALE_LOG2) {
        alpha = ptx::ex2(m_used - m_tile);
        m_used = m_tile;
    }
    // a row that has seen no key yet keeps m = -inf (general causal forms, split ranges
    // past its last key); its p must be 0
    const float neg_m = (MASK && m_used == -INFINITY) ? 0.f : -m_used;
    const uint64_t c2 = ptx::f32x2(c, c), m2 = ptx::f32x2(neg_m, neg_m);
    uint64_t acc = ptx::f32x2(0.f, 0.f);
    uint32_t pk[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        float x0, x1;
        ptx::f32x2_split(
            ptx::fma2(ptx::f32x2(__uint_as_float(s[2 * k]), __uint_as_float(s[2 * k + 1])), c2, m2),
            x0, x1);
        const float p0 = ptx::ex2(x0), p1 = ptx::ex2(x1);
        acc = ptx::add2(acc, ptx::f32x2(p0, p1));
        pk[k] = pack2<IS_BF16>(p0, p1);
    }
    float sum0, sum1;
    ptx::f32x2_split(acc, sum0, sum1);
    l = l * alpha + (sum0 + sum1);
    ptx::tmem_st32(tS, *reinterpret_cast<const uint32_t(*)[32]>(&pk[0]));
    return alpha;
}

template <bool IS_BF16, bool CAUSAL, bool NEG, bool GEN>
__device__ __forceinline__ float softmax64(uint32_t tS, int j, int kv0, int Sk, int row_vis,
                                           int tile_vis_min, float c, float& m_used, float& l) {
    const bool need_mask = (kv0 + WBN > Sk) || (CAUSAL && kv0 + WBN - 1 > tile_vis_min);
    if (need_mask) {
        int lim = Sk - 1 - kv0;
        if (CAUSAL) lim = min(lim, row_vis - kv0);
        return softmax64_body<IS_BF16, NEG, true, GEN>(tS, j, lim, c, m_used, l);
    }
    return softmax64_body<IS_BF16, NEG, false, GEN>(tS, j, 0, c, m_used, l);
}

template <int D, int NS, bool IS_BF16, bool CAUSAL, bool NEG, bool SPLIT, bool GEN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    attn_fwd_wide_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const Params p) {
    using L = Layout<D, NS>;
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
    const uint32_t B_QF = bars, B_QE = bars + 8u;
    auto B_KF = [&](int s) { return bars + 8u * (2 + s); };
    auto B_KE = [&](int s) { return bars + 8u * (2 + NS + s); };
    auto B_VF = [&](int s) { return bars + 8u * (2 + 2 * NS + s); };
    auto B_VE = [&](int s) { return bars + 8u * (2 + 3 * NS + s); };
    auto B_SF = [&](int b) { return bars + 8u * (2 + 4 * NS + b); };      // S buffer b ready
    auto B_PF = [&](int b) { return bars + 8u * (4 + 4 * NS + b); };      // P in buffer b
    const uint32_t B_PVD = bars + 8u * (6 + 4 * NS);                      // a P V finished
    const uint32_t B_OF = bars + 8u * (7 + 4 * NS);                       // last P V done
    const uint32_t B_ST = bars + 8u * (8 + 4 * NS);                       // m, l in smem
    const uint32_t B_OE = bars + 8u * (9 + 4 * NS);                       // O, m, l read
    const uint32_t B_DR = bars + 8u * (10 + 4 * NS);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
    Ctx ctx{reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4)};
    const int n_units = p.n_qp * p.BH * p.n_splits;

    if (threadIdx.x == 0) {
        ptx::mbar_init(B_QF, 1);
        ptx::mbar_init(B_QE, 1);
        for (int s = 0; s < NS; ++s) {
            ptx::mbar_init(B_KF(s), 1);
            ptx::mbar_init(B_KE(s), 1);
            ptx::mbar_init(B_VF(s), 1);
            ptx::mbar_init(B_VE(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(B_SF(b), 1);
            ptx::mbar_init(B_PF(b), 4);  // one arrival per softmax warp
        }
        ptx::mbar_init(B_PVD, 1 + 4);  // the MMA commit + one arrival per softmax warp
        ptx::mbar_init(B_OF, 1);
        ptx::mbar_init(B_ST, 4);
        ptx::mbar_init(B_OE, 4);  // one arrival per epilogue warp
        ptx::mbar_init(B_DR, 1);
        *ctx.err = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 9 && lane == 0) {
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_k);
        ptx::prefetch_tmap(&tm_v);
    }
    if (warp == 10) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < 4) {
        // ================================================================ softmax
        const int row = warp * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        const uint32_t tO = tmem + lane_base + TMEM_O;
        const float c_abs = fabsf(p.scale_log2);
        bool ok = true;
        uint32_t sfc[2] = {0, 0};  // S phases per buffer
        uint32_t gt = 0;           // KV tiles so far, all units (P V phases)
        uint32_t ut = 0;           // units with rows so far
        for (int r = 0; ok; ++r) {
            const int u = unit_of(r, n_units);
            if (u < 0) break;
            const WUnit w = decode_wunit<CAUSAL, SPLIT, GEN>(u, p);
            const int q0t = w.qt * WBM;
            const int qrow = q0t + row;
            int row_vis = qrow, tile_vis_min = q0t;
            if (GEN && w.n > 0) {
                row_vis = (p.sq_head == p.Sq ? qrow : qrow % p.sq_head) + p.causal_off;
                tile_vis_min = tile_vis<true>(q0t, min(q0t + WBM - 1, p.Sq - 1), p);
            }
            float m_used = -INFINITY, l = 0.f;
            for (int j = 0; j < w.n; ++j, ++gt) {
                const int b = j & 1;
                if (!(ok = warp_wait(ctx, B_SF(b), sfc[b] & 1))) break;
                ++sfc[b];
                // P V of global tile gt - 2 ran before S_j: see its phase complete, then
                // arrive for phase gt - 1 (see the barrier note at the top)
                if (gt >= 2 && !(ok = warp_wait(ctx, B_PVD, (gt - 2) & 1))) break;
                if (gt >= 1 && lane == 0) ptx::mbar_arrive(B_PVD);
                ptx::tc_fence_after();
                const uint32_t tS = tmem + lane_base + 64u * b;
                const float alpha = softmax64<IS_BF16, CAUSAL, NEG, GEN>(
                    tS, j, (w.kv0 + j) * WBN, p.Sk, row_vis, tile_vis_min, c_abs, m_used, l);
                if (__any_sync(0xffffffffu, alpha != 1.f)) {
                    // O holds tiles < j once P V_{j-1} has finished (it may still run:
                    // S_{j+1}, not P V_j, follows it in the MMA order)
                    if (!(ok = warp_wait(ctx, B_PVD, (gt - 1) & 1))) break;
                    ptx::tc_fence_after();
#pragma unroll 1
                    for (int cc = 0; cc < D / 32; ++cc) {
                        uint32_t ov[32];
                        ptx::tmem_ld32(tO + 32 * cc, ov);
                        ptx::tmem_wait_ld();
                        ptx::reg_fence32(ov);
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
                        ptx::tmem_st32(tO + 32 * cc, ov);
                    }
                }
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(B_PF(b));
            }
            if (!ok || w.n == 0) continue;
            if (!(ok = warp_wait(ctx, B_OE, (ut & 1) ^ 1))) break;
            s_fm[row] = m_used;
            s_fl[row] = l;
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(B_ST);
            ++ut;
        }
    } else if (warp < 8) {
        // ================================================================ epilogue
        const int wq = warp & 3;
        const int row = wq * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
        bool ok = true;
        uint32_t ut = 0;
        for (int r = 0; ok; ++r) {
            const int u = unit_of(r, n_units);
            if (u < 0) break;
            const WUnit w = decode_wunit<CAUSAL, SPLIT, GEN>(u, p);
            const int64_t head_row = static_cast<int64_t>(w.split) * p.BH + w.bh;
            const int qrow = w.qt * WBM + row;
            const bool store = qrow < p.Sq;
            if (w.n == 0) {
                if (store) write_empty_row<D, SPLIT>(p, head_row, w.bh, qrow);
                continue;
            }
            if (!(ok = warp_wait(ctx, B_ST, ut & 1))) break;
            if (!(ok = warp_wait(ctx, B_OF, ut & 1))) break;
            ptx::tc_fence_after();
            const float m_used = s_fm[row];
            const float l = s_fl[row];
            const float inv_l = l > 0.f ? 1.f / l : 0.f;
            const float lse_row =
                l > 0.f ? (m_used + log2f(l)) * 0.69314718055994530942f : -INFINITY;
            const uint32_t tO = tmem + lane_base + TMEM_O;
#pragma unroll 1
            for (int cc = 0; cc < p.d_out / 16; ++cc) {
                uint32_t ov[16];
                ptx::tmem_ld16(tO + 16 * cc, ov);
                ptx::tmem_wait_ld();
                ptx::reg_fence16(ov);
                float f0[8], f1[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    f0[e] = __uint_as_float(ov[e]) * inv_l;
                    f1[e] = __uint_as_float(ov[8 + e]) * inv_l;
                }
                if (store) {
                    store_o8<D, IS_BF16, SPLIT>(p, head_row, w.bh, qrow, 2 * cc, f0);
                    store_o8<D, IS_BF16, SPLIT>(p, head_row, w.bh, qrow, 2 * cc + 1, f1);
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(B_OE);
            ++ut;
            if (store) {
                if constexpr (SPLIT)
                    p.ws_lse[head_row * p.Sq + qrow] = lse_row;
                else if (p.lse != nullptr)
                    p.lse[static_cast<int64_t>(w.bh) * p.Sq + qrow] = lse_row;
            }
        }
    } else if (warp == 8) {
        // ================================================================ MMA issuer
        if (lane == 0) {
            constexpr uint32_t fmt = IS_BF16 ? 1u : 0u;
            constexpr uint32_t idesc_qk = ptx::idesc_f16(fmt, WBM, WBN, 0);
            constexpr uint32_t idesc_pv = ptx::idesc_f16(fmt, WBM, D, 1);
            constexpr uint32_t desc_hi = ptx::smem_desc_hi_sw128(1024);
            constexpr uint32_t KV16 = L::KV_BYTES >> 4;
            const uint32_t dq = ptx::smem_desc_lo(sQ, 16);
            const uint32_t dk0 = ptx::smem_desc_lo(sK, 16);
            const uint32_t dv0 = ptx::smem_desc_lo(sV, KV_CHUNK);
            // S_b = Q K^T for the K tile in ring slot `slot`: K steps of 16 over D,
            // +32 bytes inside a 128-byte row, +16 KB (Q) / +8 KB (K) per 64 columns
            auto issue_s = [&](int b, int slot) {
                const uint32_t kd = dk0 + static_cast<uint32_t>(slot) * KV16;
                const uint32_t d_tmem = tmem + 64u * b;
#pragma unroll
                for (int ch = 0; ch < L::NCH; ++ch) {
                    const uint32_t qa = dq + static_cast<uint32_t>(ch) * (Q_CHUNK >> 4);
                    const uint32_t kb = kd + static_cast<uint32_t>(ch) * (KV_CHUNK >> 4);
                    ptx::mma_ss_off<0, 0>(d_tmem, qa, kb, desc_hi, idesc_qk, ch > 0 ? 1u : 0u);
                    ptx::mma_ss_off<2, 2>(d_tmem, qa, kb, desc_hi, idesc_qk, 1u);
                    ptx::mma_ss_off<4, 4>(d_tmem, qa, kb, desc_hi, idesc_qk, 1u);
                    ptx::mma_ss_off<6, 6>(d_tmem, qa, kb, desc_hi, idesc_qk, 1u);
                }
                ptx::mma_commit(B_SF(b));
            };
            // O (+)= P_b V for the V tile in ring slot `slot`: K steps of 16 keys, 8 TMEM
            // columns of P and 2 KB of V each
            auto issue_pv = [&](int b, int slot, bool first) {
                const uint32_t vd = dv0 + static_cast<uint32_t>(slot) * KV16;
                const uint32_t a_tmem = tmem + 64u * b;
                const uint32_t d_tmem = tmem + TMEM_O;
                ptx::mma_ts_off<0, 0>(d_tmem, a_tmem, vd, desc_hi, idesc_pv, first ? 0u : 1u);
                ptx::mma_ts_off<8, 128>(d_tmem, a_tmem, vd, desc_hi, idesc_pv, 1u);
                ptx::mma_ts_off<16, 256>(d_tmem, a_tmem, vd, desc_hi, idesc_pv, 1u);
                ptx::mma_ts_off<24, 384>(d_tmem, a_tmem, vd, desc_hi, idesc_pv, 1u);
            };
            bool ok = true;
            uint32_t kv = 0, nu = 0, ut = 0;
            uint32_t pfc[2] = {0, 0};  // P phases per buffer
            for (int r = 0; ok; ++r) {
                const int u = unit_of(r, n_units);
                if (u < 0) break;
                const WUnit w = decode_wunit<CAUSAL, SPLIT, GEN>(u, p);
                const int n = w.n;
                if (n == 0) continue;
                auto slot = [&](int j) { return static_cast<int>((kv + j) % NS); };
                auto phase = [&](int j) { return ((kv + j) / NS) & 1u; };
                if (!(ok = wait_bounded(ctx, B_QF, nu & 1))) break;
                for (int j = 0; ok && j < 2 && j < n; ++j) {
                    if (!(ok = wait_bounded(ctx, B_KF(slot(j)), phase(j)))) break;
                    ptx::tc_fence_after();
                    issue_s(j, slot(j));
                    ptx::mma_commit(B_KE(slot(j)));
                    if (j == n - 1) ptx::mma_commit(B_QE);  // the unit's last S is issued
                }
                for (int j = 0; ok && j < n; ++j) {
                    const int b = j & 1;
                    if (!(ok = wait_bounded(ctx, B_VF(slot(j)), phase(j)))) break;
                    if (!(ok = wait_bounded(ctx, B_PF(b), pfc[b] & 1))) break;
                    ++pfc[b];
                    // the first P V of a unit overwrites O: the epilogue must have read
                    // the previous unit's O
                    if (j == 0 && !(ok = wait_bounded(ctx, B_OE, (ut & 1) ^ 1))) break;
                    ptx::tc_fence_after();
                    issue_pv(b, slot(j), j == 0);
                    ptx::mma_commit(B_VE(slot(j)));
                    ptx::mma_commit(B_PVD);
                    if (j == n - 1) ptx::mma_commit(B_OF);
                    if (j + 2 < n) {
                        if (!(ok = wait_bounded(ctx, B_KF(slot(j + 2)), phase(j + 2)))) break;
                        ptx::tc_fence_after();
                        issue_s(b, slot(j + 2));
                        ptx::mma_commit(B_KE(slot(j + 2)));
                        if (j + 2 == n - 1) ptx::mma_commit(B_QE);  // last S issued
                    }
                }
                ++ut;
                kv += static_cast<uint32_t>(n);
                ++nu;
            }
            ptx::mma_commit(B_DR);
            wait_drain(B_DR, 0);
        }
        __syncwarp();
    } else if (warp == 9) {
        // ================================================================ producer
        // Loads follow the MMA's order of use: K_0, K_1, then V_j, K_{j+2} for each j.
        if (lane == 0) {
            const bool load_q = !(p.flags & FLAG_SKIP_Q_LOAD);
            uint32_t kv = 0, nu = 0;
            int64_t last_k = -1, last_v = -1, last_q = -1;
            bool ok = true;
            auto load_kv = [&](bool is_v, uint32_t pos, int key0, int bh) {
                const int s = static_cast<int>(pos % NS);
                const uint32_t ph = (pos / NS) & 1;
                if (!wait_bounded(ctx, is_v ? B_VE(s) : B_KE(s), ph ^ 1)) return false;
                const uint32_t full = is_v ? B_VF(s) : B_KF(s);
                const uint32_t dst = (is_v ? sV : sK) + s * L::KV_BYTES;
                ptx::mbar_arrive_expect_tx(full, L::KV_BYTES);
                for (int c = 0; c < L::NCH; ++c)
                    ptx::tma_load_3d(dst + c * KV_CHUNK, is_v ? &tm_v : &tm_k, full,
                                     c * CHUNK_ELEMS, key0, bh);
                (is_v ? last_v : last_k) = pos;
                return true;
            };
            for (int r = 0; ok; ++r) {
                const int u = unit_of(r, n_units);
                if (u < 0) break;
                const WUnit w = decode_wunit<CAUSAL, SPLIT, GEN>(u, p);
                if (w.n == 0) continue;
                if (!(ok = wait_bounded(ctx, B_QE, (nu & 1) ^ 1))) break;
                if (load_q) {
                    ptx::mbar_arrive_expect_tx(B_QF, L::Q_BYTES);
                    for (int c = 0; c < L::NCH; ++c)
                        ptx::tma_load_3d(sQ + c * Q_CHUNK, &tm_q, B_QF, c * CHUNK_ELEMS,
                                         w.qt * WBM, w.bh);
                    last_q = nu;
                }
                for (int j = 0; ok && j < 2 && j < w.n; ++j)
                    ok = load_kv(false, kv + j, (w.kv0 + j) * WBN, w.bh);
                for (int j = 0; ok && j < w.n; ++j) {
                    ok = load_kv(true, kv + j, (w.kv0 + j) * WBN, w.bh);
                    if (ok && j + 2 < w.n) ok = load_kv(false, kv + j + 2, (w.kv0 + j + 2) * WBN, w.bh);
                }
                kv += static_cast<uint32_t>(w.n);
                ++nu;
            }
            // let every copy this thread started land before the CTA can exit
            if (last_q >= 0) wait_drain(B_QF, static_cast<uint32_t>(last_q) & 1);
            for (int64_t q = (last_k - NS + 1 > 0 ? last_k - NS + 1 : 0); q <= last_k; ++q)
                wait_drain(B_KF(static_cast<int>(q % NS)), (q / NS) & 1);
            for (int64_t q = (last_v - NS + 1 > 0 ? last_v - NS + 1 : 0); q <= last_v; ++q)
                wait_drain(B_VF(static_cast<int>(q % NS)), (q / NS) & 1);
        }
        __syncwarp();
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 10) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace wide
}  // namespace attn
