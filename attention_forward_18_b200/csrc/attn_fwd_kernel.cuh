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
// One CTA owns one 128-row query tile of one (batch, head) and streams the head's
// K/V in 128-key tiles:
//   warp 0      TMA producer: Q once, then K_j / V_j into a ring of NS stages
//   warp 1      MMA issuer (one thread): S_j = Q K_j^T (smem x smem -> TMEM) and
//               O += P_j V_j (P from TMEM, V from smem -> TMEM)
//   warp 2      owns the tensor-memory allocation
//   warps 4..7  softmax: thread t owns query row t of the tile; reads S_j from TMEM,
//               masks, updates the running max / normaliser, writes P_j (16-bit)
//               over S_j in TMEM, rescales O in TMEM when the max moved by more
//               than 2^8, and finally writes O / l and the LSE.
// Tensor memory (512 columns): S/P double buffer at columns 0 and 128, O at 256.
// Shared memory: Q tile + NS K tiles + NS V tiles, each tile 128 rows x D stored
// as D/64 column chunks of 128 rows x 128 bytes in the 128-byte swizzle that TMA
// writes and the tcgen05 descriptors read.
//
// Every mbarrier wait is bounded (WAIT_LIMIT_NS); on expiry the waiting role
// records ATTN_ERR_TIMEOUT in the device status word, flags the CTA, and every role
// leaves its loop, waits (again bounded) for its copies / MMAs in flight, and the
// CTA frees its tensor memory and exits.
#pragma once

#include <cuda.h>
#include <cstdint>

#include "ptx.cuh"

namespace attn {

constexpr int BM = 128;                 // query rows per tile (= TMEM lanes)
constexpr int BN = 128;                 // keys per tile
constexpr int CHUNK_ELEMS = 64;         // 16-bit elements per 128-byte swizzle row
constexpr int CHUNK_BYTES = 128 * 128;  // one chunk: 128 rows x 128 bytes
constexpr int NUM_THREADS = 256;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_S0 = 0;
constexpr uint32_t TMEM_S1 = 128;
constexpr uint32_t TMEM_O = 256;
// Lazy rescaling: the running max used for the exponentials is only moved when a
// row's new max exceeds it by more than this (log2 units); until then P can reach
// 2^8, which fp16/bf16 hold exactly in range, and O and l stay consistent because
// both are accumulated relative to the same stale max.
constexpr float LAZY_RESCALE_LOG2 = 8.0f;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;   // 2 s per wait
constexpr uint64_t DRAIN_LIMIT_NS = 500000000ull;   // 0.5 s per drain wait

constexpr int STATUS_TIMEOUT = -8;  // ATTN_ERR_TIMEOUT

// Bit 0: the producer never issues the Q load, so the MMA warp's first wait runs
// out; only the timeout test sets it.
constexpr uint32_t FLAG_SKIP_Q_LOAD = 1u;

struct Params {
    void* o;            // [BH, Sq, D] 16-bit
    float* lse;         // [BH, Sq] fp32, may be null
    int Sq, Sk, BH, n_qb;
    float scale_log2;   // scale * log2(e)
    uint32_t flags;
};

template <int D, int NS>
struct SmemLayout {
    static_assert(D % CHUNK_ELEMS == 0, "head dim must be a multiple of 64");
    static constexpr int NCH = D / CHUNK_ELEMS;
    static constexpr int TILE_BYTES = NCH * CHUNK_BYTES;  // 128 rows x D x 2 bytes
    static constexpr int Q_OFF = 0;
    static constexpr int K_OFF = Q_OFF + TILE_BYTES;
    static constexpr int V_OFF = K_OFF + NS * TILE_BYTES;
    static constexpr int BAR_OFF = V_OFF + NS * TILE_BYTES;
    // q_full, k_full[NS], k_empty[NS], v_full[NS], v_empty[NS], s_full[2],
    // p_full[2], o_done, drain
    static constexpr int NBAR = 1 + 4 * NS + 2 + 2 + 1 + 1;
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

template <int D, int NS, bool IS_BF16, bool CAUSAL>
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
    const uint32_t bars = sbase + L::BAR_OFF;
    const uint32_t B_Q = bars;
    auto B_KF = [&](int s) { return bars + 8u * (1 + s); };
    auto B_KE = [&](int s) { return bars + 8u * (1 + NS + s); };
    auto B_VF = [&](int s) { return bars + 8u * (1 + 2 * NS + s); };
    auto B_VE = [&](int s) { return bars + 8u * (1 + 3 * NS + s); };
    auto B_SF = [&](int b) { return bars + 8u * (1 + 4 * NS + b); };
    auto B_PF = [&](int b) { return bars + 8u * (3 + 4 * NS + b); };
    const uint32_t B_OD = bars + 8u * (5 + 4 * NS);
    const uint32_t B_DR = bars + 8u * (6 + 4 * NS);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
    Ctx ctx{reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4)};

    // ---- which tile: causal grids go heaviest query block first
    int qb, bh;
    if constexpr (CAUSAL) {
        qb = p.n_qb - 1 - static_cast<int>(blockIdx.x) / p.BH;
        bh = static_cast<int>(blockIdx.x) % p.BH;
    } else {
        qb = static_cast<int>(blockIdx.x) % p.n_qb;
        bh = static_cast<int>(blockIdx.x) / p.n_qb;
    }
    const int q0 = qb * BM;
    const int n_kv_all = (p.Sk + BN - 1) / BN;
    int n_kv = n_kv_all;
    if constexpr (CAUSAL) {
        const int last_row = min(q0 + BM - 1, p.Sq - 1);
        n_kv = min(n_kv_all, last_row / BN + 1);
    }

    // ---- set-up
    if (threadIdx.x == 0) {
        ptx::mbar_init(B_Q, 1);
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
        ptx::mbar_init(B_OD, 1);
        ptx::mbar_init(B_DR, 1);
        *ctx.err = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&tm_q);
        ptx::prefetch_tmap(&tm_k);
        ptx::prefetch_tmap(&tm_v);
    }
    if (warp == 2) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), TMEM_COLS);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ================================================================ producer
        if (lane == 0) {
            const bool load_q = !(p.flags & FLAG_SKIP_Q_LOAD);
            if (load_q) {
                ptx::mbar_arrive_expect_tx(B_Q, L::TILE_BYTES);
                for (int c = 0; c < L::NCH; ++c)
                    ptx::tma_load_3d(sQ + c * CHUNK_BYTES, &tm_q, B_Q, c * CHUNK_ELEMS, q0, bh);
            }
            int last_k = -1, last_v = -1;  // last issued tile index
            for (int j = 0; j < n_kv; ++j) {
                const int s = j % NS;
                const uint32_t ph = (j / NS) & 1;
                if (!wait_bounded(ctx, B_KE(s), ph ^ 1)) break;
                ptx::mbar_arrive_expect_tx(B_KF(s), L::TILE_BYTES);
                for (int c = 0; c < L::NCH; ++c)
                    ptx::tma_load_3d(sK + s * L::TILE_BYTES + c * CHUNK_BYTES, &tm_k, B_KF(s),
                                     c * CHUNK_ELEMS, j * BN, bh);
                last_k = j;
                if (!wait_bounded(ctx, B_VE(s), ph ^ 1)) break;
                ptx::mbar_arrive_expect_tx(B_VF(s), L::TILE_BYTES);
                for (int c = 0; c < L::NCH; ++c)
                    ptx::tma_load_3d(sV + s * L::TILE_BYTES + c * CHUNK_BYTES, &tm_v, B_VF(s),
                                     c * CHUNK_ELEMS, j * BN, bh);
                last_v = j;
            }
            // Let every copy this thread started land before the CTA can exit.
            if (load_q) wait_drain(B_Q, 0);
            for (int j = (last_k - NS + 1 > 0 ? last_k - NS + 1 : 0); j <= last_k; ++j)
                wait_drain(B_KF(j % NS), (j / NS) & 1);
            for (int j = (last_v - NS + 1 > 0 ? last_v - NS + 1 : 0); j <= last_v; ++j)
                wait_drain(B_VF(j % NS), (j / NS) & 1);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ================================================================ MMA issuer
        if (lane == 0) {
            constexpr uint32_t fmt = IS_BF16 ? 1u : 0u;
            constexpr uint32_t idesc_qk = ptx::idesc_f16(fmt, BM, BN, 0);
            constexpr uint32_t idesc_pv = ptx::idesc_f16(fmt, BM, D, 1);
            bool ok = wait_bounded(ctx, B_Q, 0);
            if (ok) ptx::tc_fence_after();
            for (int j = 0; ok && j <= n_kv; ++j) {
                if (j < n_kv) {
                    // S_j = Q K_j^T  (both operands K-major, 128-byte swizzle)
                    const int s = j % NS;
                    if (!(ok = wait_bounded(ctx, B_KF(s), (j / NS) & 1))) break;
                    ptx::tc_fence_after();
                    const uint32_t d_tmem = tmem + ((j & 1) ? TMEM_S1 : TMEM_S0);
                    const uint32_t kt = sK + s * L::TILE_BYTES;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk / 4) * CHUNK_BYTES + (kk % 4) * 32;
                        const uint64_t a = ptx::smem_desc_sw128(sQ + off, 16, 1024);
                        const uint64_t b = ptx::smem_desc_sw128(kt + off, 16, 1024);
                        ptx::mma_ss(d_tmem, a, b, idesc_qk, kk > 0 ? 1u : 0u);
                    }
                    ptx::mma_commit(B_SF(j & 1));
                    ptx::mma_commit(B_KE(s));
                }
                if (j >= 1) {
                    // O += P_{j-1} V_{j-1}  (P in TMEM, V MN-major in smem)
                    const int jp = j - 1;
                    const int s = jp % NS;
                    if (!(ok = wait_bounded(ctx, B_PF(jp & 1), (jp >> 1) & 1))) break;
                    if (!(ok = wait_bounded(ctx, B_VF(s), (jp / NS) & 1))) break;
                    ptx::tc_fence_after();
                    const uint32_t a_tmem = tmem + ((jp & 1) ? TMEM_S1 : TMEM_S0);
                    const uint32_t vt = sV + s * L::TILE_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk) {
                        const uint64_t b = ptx::smem_desc_sw128(vt + kk * 2048, CHUNK_BYTES, 1024);
                        ptx::mma_ts(tmem + TMEM_O, a_tmem + kk * 8, b, idesc_pv,
                                    (jp > 0 || kk > 0) ? 1u : 0u);
                    }
                    ptx::mma_commit(B_VE(s));
                    ptx::mma_commit(B_OD);
                }
            }
            // Every MMA issued above completes before the CTA frees tensor memory.
            ptx::mma_commit(B_DR);
            wait_drain(B_DR, 0);
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ================================================================ softmax
        const int wq = warp - 4;  // this warp's TMEM lane quarter
        const int row = wq * 32 + lane;
        const int qrow = q0 + row;
        const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
        const float sl2 = p.scale_log2;
        float m_used = -INFINITY;  // running max (log2 units) the exponentials use
        float l = 0.f;             // running normaliser relative to m_used
        bool ok = true;
        for (int j = 0; j < n_kv; ++j) {
            const int sb = j & 1;
            if (!(ok = warp_wait(ctx, B_SF(sb), (j >> 1) & 1))) break;
            ptx::tc_fence_after();
            const uint32_t tS = tmem + lane_base + (sb ? TMEM_S1 : TMEM_S0);
            uint32_t raw[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) ptx::tmem_ld32(tS + 32 * c, raw[c]);
            ptx::tmem_wait_ld();

            float x[128];
            const int kv0 = j * BN;
            const bool need_mask = (kv0 + BN > p.Sk) || (CAUSAL && kv0 + BN - 1 > q0);
            float mt = -INFINITY;
#pragma unroll
            for (int c = 0; c < 128; ++c) {
                float t = __uint_as_float(raw[c >> 5][c & 31]) * sl2;
                if (need_mask) {
                    const int key = kv0 + c;
                    if (key >= p.Sk || (CAUSAL && key > qrow)) t = -INFINITY;
                }
                x[c] = t;
                mt = fmaxf(mt, t);
            }
            float alpha = 1.f;
            bool rescale = false;
            if (j == 0) {
                m_used = mt;
            } else if (mt > m_used + LAZY_RESCALE_LOG2) {
                alpha = ptx::ex2(m_used - mt);
                m_used = mt;
                rescale = true;
            }
            float sum = 0.f;
            uint32_t pk[64];
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                const float p0 = ptx::ex2(x[2 * c] - m_used);
                const float p1 = ptx::ex2(x[2 * c + 1] - m_used);
                sum += p0 + p1;
                pk[c] = pack2<IS_BF16>(p0, p1);
            }
            l = l * alpha + sum;
            // P_j over S_j: 128 16-bit values = 64 columns
            ptx::tmem_st32(tS, *reinterpret_cast<const uint32_t(*)[32]>(&pk[0]));
            ptx::tmem_st32(tS + 32, *reinterpret_cast<const uint32_t(*)[32]>(&pk[32]));

            if (j > 0) {
                // O holds sum over tiles < j; PV_{j-1} must be done before touching it
                if (!(ok = warp_wait(ctx, B_OD, (j - 1) & 1))) break;
                ptx::tc_fence_after();
                if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t ov[32];
                        const uint32_t tO = tmem + lane_base + TMEM_O + 32 * c;
                        ptx::tmem_ld32(tO, ov);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
                        ptx::tmem_st32(tO, ov);
                    }
                }
            }
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(B_PF(sb));
        }

        // ---- epilogue: O / l in fp32, one rounding to 16 bits; LSE in natural log
        if (ok) ok = warp_wait(ctx, B_OD, (n_kv - 1) & 1);
        if (ok) {
            ptx::tc_fence_after();
            const float inv_l = 1.f / l;
            const bool store = qrow < p.Sq;
            uint16_t* orow = reinterpret_cast<uint16_t*>(p.o) +
                             (static_cast<int64_t>(bh) * p.Sq + qrow) * D;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t ov[32];
                ptx::tmem_ld32(tmem + lane_base + TMEM_O + 32 * c, ov);
                ptx::tmem_wait_ld();
                uint32_t packed[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    packed[e] = pack2<IS_BF16>(__uint_as_float(ov[2 * e]) * inv_l,
                                               __uint_as_float(ov[2 * e + 1]) * inv_l);
                if (store) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        dst[e] = make_uint4(packed[4 * e], packed[4 * e + 1], packed[4 * e + 2],
                                            packed[4 * e + 3]);
                }
            }
            if (store && p.lse != nullptr)
                p.lse[static_cast<int64_t>(bh) * p.Sq + qrow] =
                    (m_used + log2f(l)) * 0.69314718055994530942f;
        }
    }

    // ---- tear-down: every role is out of its loop; free tensor memory
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace attn
