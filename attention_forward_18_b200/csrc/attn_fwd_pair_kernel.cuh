// attn_fwd_pair_kernel.cuh -- the fused attention forward pass for head dimensions 192
// and 256 on a pair of CTAs (a cluster of two, one per SM) whose tensor cores run each
// MMA together (tcgen05 cta_group::2, M = 256).
//
// Why: at these D one CTA can hold only one 128-row query tile (its O takes D of the
// 512 TMEM columns), so every K/V byte it loads feeds 128 query rows, and the 64-key
// tiles that fit beside its Q make the S products N = 64 MMAs, which run into the
// per-instruction issue floor.  A pair runs a 256-row query block as one M = 256
// problem: CTA r holds query rows 128r .. 128r + 127 of the block, and of every
// 128-key tile it loads only its half of the B operands -- keys 64r .. 64r + 63 of K
// (S = Q K^T, N = 128 split over the pair) and columns (D/2)r .. (D/2)r + D/2 - 1 of V
// (O = P V, N = D split over the pair).  Per SM that halves the K/V bytes per FLOP,
// and S runs as N = 128 MMAs.  V's halves are 128 columns at D = 256 (two chunks of 64
// in the 128-byte swizzle) and 96 at D = 192 (three chunks of 32 in the 64-byte
// swizzle: a half of 96 columns does not split into 64-column chunks).
//
// Each CTA: Q (D/64 chunks of 16 KB), a ring of NSK K halves and one of NSV V halves in
// shared memory (D = 256: 3 + 2 stages of 32 KB, 224 KB with Q -- K gets the extra
// stage; D = 192: 3 + 3 stages of 24 KB); two 128-column S buffers (0, 128) and O (from
// column 256) in tensor memory.
// Rank 0 issues every MMA (S_0 S_1 | PV_0 S_2 | PV_1 S_3 | ..., KV tile j in S buffer
// j % 2); both CTAs run a TMA producer, four softmax warps (thread = row, 128 scores a
// tile) and four epilogue warps on their own rows.  Hand-offs across the pair:
//   * loads: each CTA's TMA loads count their bytes on rank 0's full barriers (rank 0's
//     producer posts the expected bytes of both halves);
//   * MMA completion (S ready, slot free, P V done, last P V): rank 0 commits to its own
//     barrier and to the same barrier of rank 1 (two commits, each with the address
//     mapped into the cluster window);
//   * P ready and O read out: rank 1's warps arrive on rank 0's barriers remotely, with
//     relaxed arrivals (what they hand over is tensor memory, ordered by the tcgen05
//     waits and fences before them; a release at cluster scope cost ~1700 clocks a tile).
// The "P V done" barrier is gated by the softmax warps as in attn_fwd_wide_kernel.cuh, so
// the softmax can rescale O while the next S runs.  Both causal forms, split ranges,
// grouped heads and negative scales as in attn_fwd_kernel.cuh; the pair always runs the
// larger of its two query tiles' KV ranges, the extra tiles fully masked for the other.
// All waits are bounded; a CTA leaves only after both CTAs of the pair are done.
#pragma once

#include "attn_fwd_kernel.cuh"

namespace attn {
namespace pair {

constexpr int NUM_THREADS = 384;
constexpr int Q_CHUNK = 128 * 128;       // 128 query rows x 128 bytes
constexpr int K_CHUNK = 64 * 128;        // 64 keys x 128 bytes (this CTA's half of a tile)
constexpr uint32_t TMEM_O = 256;         // O columns; S buffers at 0 and 128

// V halves: chunks of V_CW columns (128 keys each), MN-major in the matching swizzle.
template <int PD>
struct VGeo {
    static_assert(PD == 192 || PD == 256, "head dim 192 or 256");
    static constexpr int V_CW = PD == 256 ? 64 : 32;       // columns per chunk
    static constexpr int VCH = PD / 2 / V_CW;              // chunks per CTA (2 or 3)
    static constexpr int V_CHUNK = 128 * V_CW * 2;         // 16 KB or 8 KB
    static constexpr uint32_t SBO = 8 * V_CW * 2;          // bytes per 8-key group
    static constexpr uint32_t KSTEP = (16 * V_CW * 2) >> 4;  // 16 keys, descriptor units
};

template <int PD, int NSK, int NSV>
struct Layout {
    static constexpr int NCH = PD / CHUNK_ELEMS;        // 64-column chunks of Q and K
    static constexpr int Q_BYTES = NCH * Q_CHUNK;
    static constexpr int K_BYTES = NCH * K_CHUNK;
    static constexpr int V_BYTES = VGeo<PD>::VCH * VGeo<PD>::V_CHUNK;  // D/2 columns
    static constexpr int Q_OFF = 0;
    static constexpr int K_OFF = Q_OFF + Q_BYTES;
    static constexpr int V_OFF = K_OFF + NSK * K_BYTES;
    static constexpr int FM_OFF = V_OFF + NSV * V_BYTES;  // final max float [128]
    static constexpr int FL_OFF = FM_OFF + BM * 4;       // final sum float [128]
    static constexpr int BAR_OFF = FL_OFF + BM * 4;
    // q_full, q_empty, k_full[NSK], k_empty[NSK], v_full[NSV], v_empty[NSV], then at
    // BASE: s_full[2], p_full[2], pv_done, o_final, stats, o_free, drain
    static constexpr int BASE = 2 + 2 * NSK + 2 * NSV;
    static constexpr int NBAR = BASE + 9;
    static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
    static constexpr int BYTES = MISC_OFF + 16;
    static constexpr int ALLOC = BYTES + 1024;
    static_assert(2 * ALLOC > 232448, "one CTA per SM must be guaranteed");
    static_assert(ALLOC <= 232448, "shared memory budget exceeded");
};

// As wait_bounded / warp_wait, with acquire at cluster scope (barriers that rank 0's
// commits or the other CTA's warps arrive on).
__device__ __forceinline__ bool wait_cl(const Ctx& c, uint32_t bar, uint32_t parity) {
    if (ptx::mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    while (true) {
        if (ptx::mbar_try_wait_cluster(bar, parity)) return true;
        if (*c.err) return false;
        if (ptx::globaltimer_ns() - t0 > WAIT_LIMIT_NS) {
            raise_error(c, STATUS_TIMEOUT);
            return false;
        }
    }
}
__device__ __forceinline__ bool warp_wait_cl(const Ctx& c, uint32_t bar, uint32_t parity) {
    const bool ok = wait_cl(c, bar, parity);
    return __all_sync(0xffffffffu, ok);
}

// The r-th unit of this pair (the boustrophedon order of unit_of, over clusters).
__device__ __forceinline__ int pair_unit_of(int r, int n_units) {
    const int G = static_cast<int>(ptx::cluster_count_x());
    const int b = static_cast<int>(ptx::cluster_id_x());
    const int u = r * G + ((r & 1) ? G - 1 - b : b);
    return u < n_units ? u : -1;
}

template <int PD, int NSK, int NSV, bool IS_BF16, bool CAUSAL, bool NEG, bool SPLIT, bool GEN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    attn_fwd_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const Params p) {
    using L = Layout<PD, NSK, NSV>;
    using VG = VGeo<PD>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = ptx::smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
    const uint32_t sbase = ptx::smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = ptx::cluster_ctarank();
    const bool lead = rank == 0;

    const uint32_t sQ = sbase + L::Q_OFF;
    const uint32_t sK = sbase + L::K_OFF;
    const uint32_t sV = sbase + L::V_OFF;
    float* s_fm = reinterpret_cast<float*>(smem + L::FM_OFF);
    float* s_fl = reinterpret_cast<float*>(smem + L::FL_OFF);
    const uint32_t bars = sbase + L::BAR_OFF;
    const uint32_t B_QF = bars, B_QE = bars + 8u;
    auto B_KF = [&](int s) { return bars + 8u * (2 + s); };
    auto B_KE = [&](int s) { return bars + 8u * (2 + NSK + s); };
    auto B_VF = [&](int s) { return bars + 8u * (2 + 2 * NSK + s); };
    auto B_VE = [&](int s) { return bars + 8u * (2 + 2 * NSK + NSV + s); };
    constexpr int BA = L::BASE;
    auto B_SF = [&](int b) { return bars + 8u * (BA + b); };
    auto B_PF = [&](int b) { return bars + 8u * (BA + 2 + b); };
    const uint32_t B_PVD = bars + 8u * (BA + 4);
    const uint32_t B_OF = bars + 8u * (BA + 5);
    const uint32_t B_ST = bars + 8u * (BA + 6);
    const uint32_t B_OE = bars + 8u * (BA + 7);
    const uint32_t B_DR = bars + 8u * (BA + 8);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
    Ctx ctx{reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4)};
    const int n_units = p.n_qp * p.BH * p.n_splits;

    if (threadIdx.x == 0) {
        ptx::mbar_init(B_QF, 1);
        ptx::mbar_init(B_QE, 1);
        for (int s = 0; s < NSK; ++s) {
            ptx::mbar_init(B_KF(s), 1);
            ptx::mbar_init(B_KE(s), 1);
        }
        for (int s = 0; s < NSV; ++s) {
            ptx::mbar_init(B_VF(s), 1);
            ptx::mbar_init(B_VE(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(B_SF(b), 1);
            ptx::mbar_init(B_PF(b), 8);  // the softmax warps of both CTAs (rank 0's is used)
        }
        ptx::mbar_init(B_PVD, 1 + 4);    // rank 0's commit + this CTA's softmax warps
        ptx::mbar_init(B_OF, 1);
        ptx::mbar_init(B_ST, 4);
        ptx::mbar_init(B_OE, lead ? 8 : 4);  // rank 0: the epilogue warps of both CTAs
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
        ptx::tmem_alloc_pair(ptx::smem_u32(tmem_slot), TMEM_COLS);
        ptx::tmem_relinquish_pair();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();  // both CTAs' barriers exist before either signals the other's
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // Registers: the launch gives 384 threads x 168; the softmax warpgroup holds a row's
    // 128 scores and their 64 packed pairs, the others little:
    // 128 x 216 + 128 x 136 + 128 x 136 = 62464 <= 64512.
    if (warp < 4) {
        // ================================================================ softmax
        ptx::setmaxnreg_inc<216>();
        const int row = warp * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        const uint32_t tO = tmem + lane_base + TMEM_O;
        const uint32_t pf_remote[2] = {ptx::mapa_shared(B_PF(0), 0), ptx::mapa_shared(B_PF(1), 0)};
        const float c_abs = fabsf(p.scale_log2);
        bool ok = true;
        uint32_t sfc[2] = {0, 0};
        uint32_t gt = 0;
        uint32_t ut = 0;
        for (int r = 0; ok; ++r) {
            const int u = pair_unit_of(r, n_units);
            if (u < 0) break;
            const Unit w = decode_unit<CAUSAL, SPLIT, GEN>(u, p);
            const int n = max(w.n[0], w.n[1]);
            if (n == 0) continue;
            const int q0t = w.qp * ROWS_PER_CTA + BM * static_cast<int>(rank);
            const int qrow = q0t + row;
            int row_vis = qrow, tile_vis_min = q0t;
            if (GEN) {
                row_vis = (p.sq_head == p.Sq ? qrow : qrow % p.sq_head) + p.causal_off;
                tile_vis_min = tile_vis<true>(q0t, min(q0t + BM - 1, p.Sq - 1), p);
            }
            float m_used = -INFINITY;
            float l = 0.f;
            for (int j = 0; j < n; ++j, ++gt) {
                const int b = j & 1;
                if (!(ok = warp_wait_cl(ctx, B_SF(b), sfc[b] & 1))) break;
                ++sfc[b];
                // P V of global tile gt - 2 ran before S_j: see its phase complete, then
                // arrive for phase gt - 1 (the gating of attn_fwd_wide_kernel.cuh)
                if (gt >= 2 && !(ok = warp_wait_cl(ctx, B_PVD, (gt - 2) & 1))) break;
                if (gt >= 1 && lane == 0) ptx::mbar_arrive(B_PVD);
                ptx::tc_fence_after();
                // (the pair runs the larger KV range of its two query tiles, so causal rows
                // can meet tiles, even a first tile, with no visible key: keep the guard)
                // (a row-sum limit of 2^8: a jump in a row's max by more than the lazy
                // threshold always leaves its dominant p exactly 1)
                const float alpha = softmax_tile<IS_BF16, CAUSAL, NEG, CAUSAL, 8>(
                    tmem + lane_base + 128u * b, j, (w.kv0 + j) * BN, p.Sk, row_vis,
                    tile_vis_min, c_abs, m_used, l);
                if (__any_sync(0xffffffffu, alpha != 1.f)) {
                    if (!(ok = warp_wait_cl(ctx, B_PVD, (gt - 1) & 1))) break;
                    ptx::tc_fence_after();
#pragma unroll 1
                    for (int cc = 0; cc < PD / 32; ++cc) {
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
                if (lane == 0) {
                    if (lead) ptx::mbar_arrive(B_PF(b));
                    else ptx::mbar_arrive_cluster_relaxed(pf_remote[b]);
                }
            }
            if (!ok) continue;
            if (!(ok = warp_wait_cl(ctx, B_OE, (ut & 1) ^ 1))) break;
            s_fm[row] = m_used;
            s_fl[row] = l;
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(B_ST);
            ++ut;
        }
    } else if (warp < 8) {
        // ================================================================ epilogue
        ptx::setmaxnreg_dec<136>();
        const int wq = warp & 3;
        const int row = wq * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t oe_remote = ptx::mapa_shared(B_OE, 0);
        bool ok = true;
        uint32_t ut = 0;
        for (int r = 0; ok; ++r) {
            const int u = pair_unit_of(r, n_units);
            if (u < 0) break;
            const Unit w = decode_unit<CAUSAL, SPLIT, GEN>(u, p);
            const int64_t head_row = static_cast<int64_t>(w.split) * p.BH + w.bh;
            const int qrow = w.qp * ROWS_PER_CTA + BM * static_cast<int>(rank) + row;
            const bool store = qrow < p.Sq;
            if (max(w.n[0], w.n[1]) == 0) {
                if (store) write_empty_row<PD, SPLIT>(p, head_row, w.bh, qrow);
                continue;
            }
            if (!(ok = warp_wait(ctx, B_ST, ut & 1))) break;
            if (!(ok = warp_wait_cl(ctx, B_OF, ut & 1))) break;
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
                    store_o8<PD, IS_BF16, SPLIT>(p, head_row, w.bh, qrow, 2 * cc, f0);
                    store_o8<PD, IS_BF16, SPLIT>(p, head_row, w.bh, qrow, 2 * cc + 1, f1);
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                ptx::mbar_arrive(B_OE);
                if (!lead) ptx::mbar_arrive_cluster_relaxed(oe_remote);
            }
            ++ut;
            if (store) {
                if constexpr (SPLIT)
                    p.ws_lse[head_row * p.Sq + qrow] = lse_row;
                else if (p.lse != nullptr)
                    p.lse[static_cast<int64_t>(w.bh) * p.Sq + qrow] = lse_row;
            }
        }
    } else {
        ptx::setmaxnreg_dec<136>();
    if (warp == 8) {
        // ================================================================ MMA issuer (rank 0)
        if (lead && lane == 0) {
            constexpr uint32_t fmt = IS_BF16 ? 1u : 0u;
            constexpr uint32_t idesc_qk = ptx::idesc_f16(fmt, 2 * BM, BN, 0);
            constexpr uint32_t idesc_pv = ptx::idesc_f16(fmt, 2 * BM, PD, 1);
            constexpr uint32_t desc_hi = ptx::smem_desc_hi_sw128(1024);
            constexpr uint32_t v_hi = PD == 256 ? ptx::smem_desc_hi_sw128(VG::SBO)
                                                : ptx::smem_desc_hi_sw64(VG::SBO);
            const uint32_t dq = ptx::smem_desc_lo(sQ, 16);
            const uint32_t dk0 = ptx::smem_desc_lo(sK, 16);
            const uint32_t dv0 = ptx::smem_desc_lo(sV, VG::V_CHUNK);
            // completion to this CTA's barrier and to the same barrier of rank 1
            auto commit2 = [&](uint32_t bar) {
                ptx::mma_commit_pair(bar);
                ptx::mma_commit_pair(ptx::mapa_shared(bar, 1));
            };
            // S_b = Q K^T (M = 256, N = 128 keys): K steps of 16 over D
            auto issue_s = [&](int b, int slot) {
                const uint32_t kd = dk0 + static_cast<uint32_t>(slot) * (L::K_BYTES >> 4);
                const uint32_t d_tmem = tmem + 128u * b;
#pragma unroll
                for (int ch = 0; ch < L::NCH; ++ch) {
                    const uint32_t qa = dq + static_cast<uint32_t>(ch) * (Q_CHUNK >> 4);
                    const uint32_t kb = kd + static_cast<uint32_t>(ch) * (K_CHUNK >> 4);
                    ptx::mma2_ss_off<0, 0>(d_tmem, qa, kb, desc_hi, idesc_qk, ch > 0 ? 1u : 0u);
                    ptx::mma2_ss_off<2, 2>(d_tmem, qa, kb, desc_hi, idesc_qk, 1u);
                    ptx::mma2_ss_off<4, 4>(d_tmem, qa, kb, desc_hi, idesc_qk, 1u);
                    ptx::mma2_ss_off<6, 6>(d_tmem, qa, kb, desc_hi, idesc_qk, 1u);
                }
                commit2(B_SF(b));
            };
            // O (+)= P_b V (M = 256, N = D): K steps of 16 keys, 8 TMEM columns of P and
            // 16 rows of each V chunk
            auto issue_pv = [&](int b, int slot, bool first) {
                constexpr uint32_t K1 = VG::KSTEP;
                const uint32_t vd = dv0 + static_cast<uint32_t>(slot) * (L::V_BYTES >> 4);
                const uint32_t a_tmem = tmem + 128u * b;
                const uint32_t d_tmem = tmem + TMEM_O;
                ptx::mma2_ts_off<0, 0>(d_tmem, a_tmem, vd, v_hi, idesc_pv, first ? 0u : 1u);
                ptx::mma2_ts_off<8, K1>(d_tmem, a_tmem, vd, v_hi, idesc_pv, 1u);
                ptx::mma2_ts_off<16, 2 * K1>(d_tmem, a_tmem, vd, v_hi, idesc_pv, 1u);
                ptx::mma2_ts_off<24, 3 * K1>(d_tmem, a_tmem, vd, v_hi, idesc_pv, 1u);
                ptx::mma2_ts_off<32, 4 * K1>(d_tmem, a_tmem, vd, v_hi, idesc_pv, 1u);
                ptx::mma2_ts_off<40, 5 * K1>(d_tmem, a_tmem, vd, v_hi, idesc_pv, 1u);
                ptx::mma2_ts_off<48, 6 * K1>(d_tmem, a_tmem, vd, v_hi, idesc_pv, 1u);
                ptx::mma2_ts_off<56, 7 * K1>(d_tmem, a_tmem, vd, v_hi, idesc_pv, 1u);
            };
            bool ok = true;
            uint32_t kv = 0, nu = 0, ut = 0;
            uint32_t pfc[2] = {0, 0};
            for (int r = 0; ok; ++r) {
                const int u = pair_unit_of(r, n_units);
                if (u < 0) break;
                const Unit w = decode_unit<CAUSAL, SPLIT, GEN>(u, p);
                const int n = max(w.n[0], w.n[1]);
                if (n == 0) continue;
                auto kslot = [&](int j) { return static_cast<int>((kv + j) % NSK); };
                auto kphase = [&](int j) { return ((kv + j) / NSK) & 1u; };
                auto vslot = [&](int j) { return static_cast<int>((kv + j) % NSV); };
                auto vphase = [&](int j) { return ((kv + j) / NSV) & 1u; };
                if (!(ok = wait_cl(ctx, B_QF, nu & 1))) break;
                for (int j = 0; ok && j < 2 && j < n; ++j) {
                    if (!(ok = wait_cl(ctx, B_KF(kslot(j)), kphase(j)))) break;
                    ptx::tc_fence_after();
                    issue_s(j, kslot(j));
                    commit2(B_KE(kslot(j)));
                    if (j == n - 1) commit2(B_QE);  // the unit's last S is issued
                }
                for (int j = 0; ok && j < n; ++j) {
                    const int b = j & 1;
                    if (!(ok = wait_cl(ctx, B_VF(vslot(j)), vphase(j)))) break;
                    if (!(ok = wait_cl(ctx, B_PF(b), pfc[b] & 1))) break;
                    ++pfc[b];
                    // the first P V of a unit overwrites O: both epilogues must have read
                    // the previous unit's O
                    if (j == 0 && !(ok = wait_cl(ctx, B_OE, (ut & 1) ^ 1))) break;
                    ptx::tc_fence_after();
                    issue_pv(b, vslot(j), j == 0);
                    commit2(B_VE(vslot(j)));
                    commit2(B_PVD);
                    if (j == n - 1) commit2(B_OF);
                    if (j + 2 < n) {
                        if (!(ok = wait_cl(ctx, B_KF(kslot(j + 2)), kphase(j + 2)))) break;
                        ptx::tc_fence_after();
                        issue_s(b, kslot(j + 2));
                        commit2(B_KE(kslot(j + 2)));
                        if (j + 2 == n - 1) commit2(B_QE);
                    }
                }
                ++ut;
                kv += static_cast<uint32_t>(n);
                ++nu;
            }
            ptx::mma_commit_pair(B_DR);
            wait_drain(B_DR, 0);
        }
        __syncwarp();
    } else if (warp == 9) {
        // ================================================================ producers
        // Both CTAs load their halves (K_0 .. K_{NSK-1}, then V_j, K_{j+NSK}), the bytes
        // counted on rank 0's full barriers; rank 0 posts the expected bytes of both
        // halves.  The tensor maps see each operand as (chunk columns, rows, column
        // chunk, head), so one box lands a whole half tile chunk-major: Q 128 rows and K
        // 64 keys x D/64 chunks of 64 columns, V 128 keys x this CTA's chunks.
        if (lane == 0) {
            const bool load_q = !(p.flags & FLAG_SKIP_Q_LOAD);
            const int rk = static_cast<int>(rank);
            uint32_t kv = 0, nu = 0;
            int64_t last_k = -1, last_v = -1, last_q = -1;
            bool ok = true;
            auto load_k = [&](uint32_t pos, int kt, int bh) {
                const int s = static_cast<int>(pos % NSK);
                if (!wait_cl(ctx, B_KE(s), ((pos / NSK) & 1) ^ 1)) return false;
                if (lead) ptx::mbar_arrive_expect_tx(B_KF(s), 2 * L::K_BYTES);
                ptx::tma_load_4d_pair(sK + s * L::K_BYTES, &tm_k, ptx::mapa_shared(B_KF(s), 0), 0,
                                      kt * BN + 64 * rk, 0, bh);
                last_k = pos;
                return true;
            };
            auto load_v = [&](uint32_t pos, int kt, int bh) {
                const int s = static_cast<int>(pos % NSV);
                if (!wait_cl(ctx, B_VE(s), ((pos / NSV) & 1) ^ 1)) return false;
                if (lead) ptx::mbar_arrive_expect_tx(B_VF(s), 2 * L::V_BYTES);
                ptx::tma_load_4d_pair(sV + s * L::V_BYTES, &tm_v, ptx::mapa_shared(B_VF(s), 0), 0,
                                      kt * BN, VG::VCH * rk, bh);
                last_v = pos;
                return true;
            };
            for (int r = 0; ok; ++r) {
                const int u = pair_unit_of(r, n_units);
                if (u < 0) break;
                const Unit w = decode_unit<CAUSAL, SPLIT, GEN>(u, p);
                const int n = max(w.n[0], w.n[1]);
                if (n == 0) continue;
                if (!(ok = wait_cl(ctx, B_QE, (nu & 1) ^ 1))) break;
                if (load_q) {
                    if (lead) ptx::mbar_arrive_expect_tx(B_QF, 2 * L::Q_BYTES);
                    ptx::tma_load_4d_pair(sQ, &tm_q, ptx::mapa_shared(B_QF, 0), 0,
                                          w.qp * ROWS_PER_CTA + BM * rk, 0, w.bh);
                    last_q = nu;
                }
                // K runs NSK tiles ahead: K_{j+NSK} waits only for S_j, not behind V_j's
                // slot (freed by P V_{j-2})
                for (int j = 0; ok && j < NSK && j < n; ++j) ok = load_k(kv + j, w.kv0 + j, w.bh);
                for (int j = 0; ok && j < n; ++j) {
                    ok = load_v(kv + j, w.kv0 + j, w.bh);
                    if (ok && j + NSK < n) ok = load_k(kv + j + NSK, w.kv0 + j + NSK, w.bh);
                }
                kv += static_cast<uint32_t>(n);
                ++nu;
            }
            // rank 0's full barriers count both CTAs' bytes: once they complete, every
            // copy of the pair has landed (rank 1 leaves only after rank 0, below)
            if (lead) {
                if (last_q >= 0) wait_drain(B_QF, static_cast<uint32_t>(last_q) & 1);
                for (int64_t q = (last_k - NSK + 1 > 0 ? last_k - NSK + 1 : 0); q <= last_k; ++q)
                    wait_drain(B_KF(static_cast<int>(q % NSK)), (q / NSK) & 1);
                for (int64_t q = (last_v - NSV + 1 > 0 ? last_v - NSV + 1 : 0); q <= last_v; ++q)
                    wait_drain(B_VF(static_cast<int>(q % NSV)), (q / NSV) & 1);
            }
        }
        __syncwarp();
    }
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::cluster_sync();  // neither CTA leaves while the pair's MMAs, copies or arrivals run
    if (warp == 10) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc_pair(tmem, TMEM_COLS);
    }
}

}  // namespace pair
}  // namespace attn
