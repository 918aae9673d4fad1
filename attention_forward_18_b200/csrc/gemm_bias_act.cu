// gemm_bias_act.cu -- C = act(A W^T + bias) on the sm_100a tensor cores, the C ABI of
// include/gemm_bias_act.h.
//
// Persistent, warp-specialised, one CTA per SM (384 threads):
//   warp 0       TMA producer: 128x64 tiles of A and 256x64 tiles of W (128-byte
//                swizzle) into a 4-stage shared-memory ring (48 KB per stage);
//   warp 1       MMA issuer: per 64-wide K block four tcgen05.mma (M=128, N=256,
//                K=16) into one of two fp32 accumulators in tensor memory (2 x 256
//                columns), so the epilogue of one tile overlaps the products of the
//                next;
//   warp 2       tensor-memory allocation / release;
//   warps 4..11  epilogue: tcgen05.ld of the accumulator (warp w reads TMEM lane
//                quarter w % 4, column half (w - 4) / 4), + bias, activation in fp32
//                (GELU through a published rational-exponential form of erf), one
//                rounding to 16 bits, 16-byte stores.
// Output tiles are visited in groups of 8 M-blocks (N-blocks inner within a group) so
// the CTAs running at one time share their A and W tiles in L2.
// Every wait is bounded (2 s); a timeout records ATTN_ERR_TIMEOUT in this file's
// status word (read through attn_fwd_status), all roles leave their loops, in-flight
// copies and MMAs are drained (bounded) and tensor memory is freed.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <climits>
#include <cstdint>
#include <mutex>

#include "attn_fwd.h"
#include "gemm_bias_act.h"
#include "ptx.cuh"

namespace gemm {

namespace ptx = attn::ptx;

constexpr int BN = 256, BK = 64;
constexpr int B_BYTES = BN * BK * 2;           // 32 KB
constexpr int EPI_WARP0 = 4;
constexpr int GROUP_M = 8;
constexpr uint32_t TMEM_COLS = 512;

// Tile shapes.  MH = 1: 128 x 256 tiles, a 4-stage ring of 48 KB, two 256-column
// accumulators (the epilogue of one tile overlaps the next tile's products).  MH = 2:
// 256 x 256 tiles as two M = 128 halves sharing each W tile, a 3-stage ring of 64 KB,
// one accumulator of two halves (all 512 columns), so a third less A/W traffic per
// FLOP at the price of an epilogue the next tile waits for (used for long K).
template <int MH>
struct Cfg {
    static constexpr int BM = 128 * MH;
    static constexpr int STAGES = MH == 1 ? 4 : 3;
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int EPI_WARPS = 8 * MH;
    static constexpr int NUM_THREADS = 32 * (EPI_WARP0 + EPI_WARPS);
    static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
    // full[STAGES], empty[STAGES], acc_full[2], acc_empty[2], drain
    static constexpr int NBAR = 2 * STAGES + 5;
    static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
    static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;  // + slack to align to 1024
    static_assert(2 * SMEM_BYTES > 232448, "one CTA per SM (it takes all of TMEM)");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;
constexpr uint64_t DRAIN_LIMIT_NS = 500000000ull;
constexpr int STATUS_TIMEOUT = -8;             // ATTN_ERR_TIMEOUT


struct Params {
    void* c;              // [M, N] 16-bit
    const void* bias;     // [N] 16-bit or null
    int M, N, K;
    int num_m, num_n, num_k, num_tiles;
    uint32_t flags;       // bit 0: the producer skips its loads (timeout test)
};

__device__ int g_gemm_status;

struct Ctx {
    volatile int* err;
};

__device__ __forceinline__ void raise_error(const Ctx& c, int code) {
    *c.err = 1;
    atomicCAS(&g_gemm_status, 0, code);
}

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

__device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = ptx::globaltimer_ns();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (ptx::globaltimer_ns() - t0 > DRAIN_LIMIT_NS) return false;
    }
    return true;
}

__device__ __forceinline__ bool warp_wait(const Ctx& c, uint32_t bar, uint32_t parity) {
    const bool ok = wait_bounded(c, bar, parity);
    return __all_sync(0xffffffffu, ok);
}

// Output tile t -> (M-block, N-block): groups of GROUP_M M-blocks, N-blocks outer
// within a group.
__device__ __forceinline__ void tile_coords(int t, const Params& p, int& mb, int& nb) {
    const int per_group = GROUP_M * p.num_n;
    const int g = t / per_group;
    const int first = g * GROUP_M;
    const int rows = min(p.num_m - first, GROUP_M);
    const int r = t - g * per_group;
    mb = first + r % rows;
    nb = r / rows;
}

__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// GELU(z) = 0.5 z (1 + erf(z / sqrt 2)) with erf from Abramowitz and Stegun, formula
// 7.1.26: for x >= 0, erf(x) = 1 - (a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5) e^(-x^2),
// t = 1 / (1 + p x), absolute error <= 1.5e-7.  The bracket is erfc(x), so for z < 0
// the factor 1 + erf = erfc(|x|) comes without cancellation; for z >= 0 it is 2 - erfc.
// Absolute error of the result <= 0.5 |z| (1.5e-7 + a few fp32 roundings).
__device__ __forceinline__ float gelu(float z) {
    const float x = fabsf(z) * 0.70710678118654752f;
    const float t = rcp_approx(fmaf(0.3275911f, x, 1.f));
    float poly = fmaf(1.061405429f, t, -1.453152027f);
    poly = fmaf(poly, t, 1.421413741f);
    poly = fmaf(poly, t, -0.284496736f);
    poly = fmaf(poly, t, 0.254829592f) * t;
    const float erfc_x = poly * ptx::ex2(-x * x * 1.4426950408889634f);
    return 0.5f * z * (z >= 0.f ? 2.f - erfc_x : erfc_x);
}

template <int ACT>
__device__ __forceinline__ float activate(float z) {
    if constexpr (ACT == GEMM_ACT_GELU) return gelu(z);
    else if constexpr (ACT == GEMM_ACT_RELU) return fmaxf(z, 0.f);
    else return z;
}

// The low / high 16-bit value of a packed pair, as fp32.
template <bool IS_BF16>
__device__ __forceinline__ float unpack_lo(uint32_t w) {
    if constexpr (IS_BF16) return __uint_as_float(w << 16);
    else return __half2float(__ushort_as_half(static_cast<uint16_t>(w & 0xffffu)));
}
template <bool IS_BF16>
__device__ __forceinline__ float unpack_hi(uint32_t w) {
    if constexpr (IS_BF16) return __uint_as_float(w & 0xffff0000u);
    else return __half2float(__ushort_as_half(static_cast<uint16_t>(w >> 16)));
}

template <bool IS_BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    if constexpr (IS_BF16) return ptx::pack_bf16x2(lo, hi);
    else return ptx::pack_f16x2(lo, hi);
}

template <bool IS_BF16, int ACT, bool HAS_BIAS, int MH>
__global__ void __launch_bounds__(Cfg<MH>::NUM_THREADS, 1)
    gemm_bias_act_kernel(const __grid_constant__ CUtensorMap tm_a,
                         const __grid_constant__ CUtensorMap tm_w, const Params p) {
    using C = Cfg<MH>;
    constexpr int BM = C::BM, STAGES = C::STAGES, A_BYTES = C::A_BYTES;
    constexpr int STAGE_BYTES = C::STAGE_BYTES, EPI_WARPS = C::EPI_WARPS;
    constexpr int BAR_OFF = C::BAR_OFF, MISC_OFF = C::MISC_OFF;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = ptx::smem_u32(smem_raw);
    uint8_t* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
    const uint32_t sbase = ptx::smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const uint32_t bars = sbase + BAR_OFF;
    auto B_FULL = [&](int s) { return bars + 8u * s; };
    auto B_EMPTY = [&](int s) { return bars + 8u * (STAGES + s); };
    auto B_AF = [&](int b) { return bars + 8u * (2 * STAGES + b); };      // accumulator b done
    auto B_AE = [&](int b) { return bars + 8u * (2 * STAGES + 2 + b); };  // accumulator b read
    const uint32_t B_DR = bars + 8u * (2 * STAGES + 4);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + MISC_OFF);
    Ctx ctx{reinterpret_cast<volatile int*>(smem + MISC_OFF + 4)};

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            ptx::mbar_init(B_FULL(s), 1);
            ptx::mbar_init(B_EMPTY(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(B_AF(b), 1);
            ptx::mbar_init(B_AE(b), EPI_WARPS);
        }
        ptx::mbar_init(B_DR, 1);
        *ctx.err = 0;
        ptx::fence_mbar_init();
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
        // ================================================================ TMA producer
        if (lane == 0) {
            ptx::prefetch_tmap(&tm_a);
            ptx::prefetch_tmap(&tm_w);
            const bool load = !(p.flags & 1u);
            uint32_t it = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x) {
                int mb, nb;
                tile_coords(t, p, mb, nb);
                for (int kb = 0; kb < p.num_k; ++kb, ++it) {
                    const int s = static_cast<int>(it % STAGES);
                    const uint32_t ph = (it / STAGES) & 1u;
                    if (!(ok = wait_bounded(ctx, B_EMPTY(s), ph ^ 1u))) break;
                    if (!load) continue;
                    const uint32_t sa = sbase + s * STAGE_BYTES;
                    ptx::mbar_arrive_expect_tx(B_FULL(s), STAGE_BYTES);
                    ptx::tma_load_2d(sa, &tm_a, B_FULL(s), kb * BK, mb * BM);
                    ptx::tma_load_2d(sa + A_BYTES, &tm_w, B_FULL(s), kb * BK, nb * BN);
                }
            }
            // let the copies in flight land before the CTA can exit
            if (load) {
                const uint32_t n = it < STAGES ? it : STAGES;
                for (uint32_t q = it - n; q < it; ++q)
                    wait_drain(B_FULL(static_cast<int>(q % STAGES)), (q / STAGES) & 1u);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ================================================================ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = ptx::idesc_f16(IS_BF16 ? 1u : 0u, 128, BN, 0);
            constexpr uint32_t hi = ptx::smem_desc_hi_sw128(1024);
            uint32_t it = 0, i = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x, ++i) {
                // MH = 1: accumulator i % 2, used every other tile; MH = 2: the one
                // accumulator (both halves), used every tile
                const int ab = MH == 1 ? static_cast<int>(i & 1u) : 0;
                const uint32_t use = MH == 1 ? (i >> 1) : i;
                if (!(ok = wait_bounded(ctx, B_AE(ab), (use & 1u) ^ 1u))) break;
                ptx::tc_fence_after();
                for (int kb = 0; kb < p.num_k; ++kb, ++it) {
                    const int s = static_cast<int>(it % STAGES);
                    if (!(ok = wait_bounded(ctx, B_FULL(s), (it / STAGES) & 1u))) break;
                    ptx::tc_fence_after();
                    const uint32_t sa = sbase + s * STAGE_BYTES;
                    const uint32_t b_lo = ptx::smem_desc_lo(sa + A_BYTES, 16);
#pragma unroll
                    for (int h = 0; h < MH; ++h) {
                        // half h: rows 128h.. of the A tile (16 KB further), columns
                        // 256(ab + h) of tensor memory
                        const uint32_t d = tmem + static_cast<uint32_t>(ab + h) * BN;
                        const uint32_t a_lo = ptx::smem_desc_lo(sa + h * 16384, 16);
                        // K steps of 16 elements: +32 bytes inside the 128-byte row
                        ptx::mma_ss_off<0, 0>(d, a_lo, b_lo, hi, idesc, kb > 0 ? 1u : 0u);
                        ptx::mma_ss_off<2, 2>(d, a_lo, b_lo, hi, idesc, 1u);
                        ptx::mma_ss_off<4, 4>(d, a_lo, b_lo, hi, idesc, 1u);
                        ptx::mma_ss_off<6, 6>(d, a_lo, b_lo, hi, idesc, 1u);
                    }
                    ptx::mma_commit(B_EMPTY(s));
                }
                if (!ok) break;
                ptx::mma_commit(B_AF(ab));
            }
            // every MMA issued above completes before tensor memory is freed
            ptx::mma_commit(B_DR);
            wait_drain(B_DR, 0);
        }
        __syncwarp();
    } else if (warp >= EPI_WARP0) {
        // ================================================================ epilogue
        const bool bias_vec = (reinterpret_cast<uintptr_t>(p.bias) & 15u) == 0;
        const int q = warp & 3;                          // TMEM lane quarter
        const int half = ((warp - EPI_WARP0) >> 2) & 1;  // column half of the tile
        const int mh = (warp - EPI_WARP0) >> 3;          // MH = 2: the M half
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        uint32_t i = 0;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x, ++i) {
            int mb, nb;
            tile_coords(t, p, mb, nb);
            const int ab = MH == 1 ? static_cast<int>(i & 1u) : 0;
            const uint32_t use = MH == 1 ? (i >> 1) : i;
            if (!(ok = warp_wait(ctx, B_AF(ab), use & 1u))) break;
            ptx::tc_fence_after();
            const int row = mb * BM + mh * 128 + q * 32 + lane;
            const bool row_ok = row < p.M;
            uint16_t* crow = reinterpret_cast<uint16_t*>(p.c) + static_cast<int64_t>(row) * p.N;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                const int col0 = nb * BN + half * 128 + c * 32;
                uint32_t v[32];
                ptx::tmem_ld32(tmem + lane_base +
                                   static_cast<uint32_t>((ab + mh) * BN + half * 128 + c * 32), v);
                ptx::tmem_wait_ld();
                ptx::reg_fence32(v);
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const int cg = col0 + 8 * g;  // N is a multiple of 8: groups are whole
                    if (cg >= p.N) continue;
                    uint32_t w[4];
                    // the group's 8 bias values: one 16-byte load when the bias is
                    // 16-byte aligned (cg is a multiple of 8), else one by one
                    uint32_t bw[4] = {0u, 0u, 0u, 0u};
                    if constexpr (HAS_BIAS) {
                        if (bias_vec) {
                            const uint4 bv = *reinterpret_cast<const uint4*>(
                                reinterpret_cast<const uint16_t*>(p.bias) + cg);
                            bw[0] = bv.x, bw[1] = bv.y, bw[2] = bv.z, bw[3] = bv.w;
                        } else {
                            const uint16_t* bp = reinterpret_cast<const uint16_t*>(p.bias) + cg;
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                bw[e] = static_cast<uint32_t>(bp[2 * e]) |
                                        (static_cast<uint32_t>(bp[2 * e + 1]) << 16);
                        }
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float z0 = __uint_as_float(v[8 * g + 2 * e]);
                        float z1 = __uint_as_float(v[8 * g + 2 * e + 1]);
                        if constexpr (HAS_BIAS) {
                            z0 += unpack_lo<IS_BF16>(bw[e]);
                            z1 += unpack_hi<IS_BF16>(bw[e]);
                        }
                        w[e] = pack2<IS_BF16>(activate<ACT>(z0), activate<ACT>(z1));
                    }
                    if (row_ok)
                        *reinterpret_cast<uint4*>(crow + cg) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            // the accumulator is read: the MMA warp may start the tile after next in it
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(B_AE(ab));
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace gemm

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// [rows, K] 16-bit row-major as a 2-D tensor (K innermost); box 64 x box_rows with
// the 128-byte swizzle; out-of-range rows / columns read as zeros.
bool encode_2d(CUtensorMap* m, const void* base, int K, int rows, int box_rows, bool bf16) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(gemm::BK),
                               static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
              const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int device_sms() {
    static int sms[64];
    static std::mutex mu;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return -1;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (sms[dev] == 0) {
        int major = 0, n = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return -1;
        }
        sms[dev] = (major == 10 && n > 0) ? n : -1;
    }
    return sms[dev];
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

template <bool BF16, int ACT, bool BIAS, int MH>
int launch(const CUtensorMap& ta, const CUtensorMap& tw, const gemm::Params& p, int grid,
           cudaStream_t s) {
    using C = gemm::Cfg<MH>;
    auto k = gemm::gemm_bias_act_kernel<BF16, ACT, BIAS, MH>;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
        cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_LAUNCH;
    }
    k<<<grid, C::NUM_THREADS, C::SMEM_BYTES, s>>>(ta, tw, p);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

template <bool BF16, int ACT, int MH>
int launch_bias(const CUtensorMap& ta, const CUtensorMap& tw, const gemm::Params& p, int grid,
                cudaStream_t s) {
    return p.bias ? launch<BF16, ACT, true, MH>(ta, tw, p, grid, s)
                  : launch<BF16, ACT, false, MH>(ta, tw, p, grid, s);
}

template <bool BF16, int MH>
int launch_act(const CUtensorMap& ta, const CUtensorMap& tw, const gemm::Params& p, int act,
               int grid, cudaStream_t s) {
    if (act == GEMM_ACT_GELU) return launch_bias<BF16, GEMM_ACT_GELU, MH>(ta, tw, p, grid, s);
    if (act == GEMM_ACT_RELU) return launch_bias<BF16, GEMM_ACT_RELU, MH>(ta, tw, p, grid, s);
    return launch_bias<BF16, GEMM_ACT_NONE, MH>(ta, tw, p, grid, s);
}

int run(const void* a, const void* w, const void* bias, void* c, int M, int N, int K, int act,
        int dtype, cudaStream_t stream, unsigned flags) {
    if (!a || !w || !c) return ATTN_ERR_NULLPTR;
    if (dtype != ATTN_F16 && dtype != ATTN_BF16) return ATTN_ERR_DTYPE;
    if (act != GEMM_ACT_NONE && act != GEMM_ACT_GELU && act != GEMM_ACT_RELU) return ATTN_ERR_SHAPE;
    if (M < 1 || N < 1 || K < 1 || N % 8 != 0 || K % 8 != 0) return ATTN_ERR_SHAPE;
    auto mis16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) != 0; };
    if (mis16(a) || mis16(w) || mis16(c)) return ATTN_ERR_ALIGN;
    if (bias && (reinterpret_cast<uintptr_t>(bias) & 1u)) return ATTN_ERR_ALIGN;
    const size_t na = static_cast<size_t>(M) * K * 2, nw = static_cast<size_t>(N) * K * 2;
    const size_t nc = static_cast<size_t>(M) * N * 2;
    if (overlaps(c, nc, a, na) || overlaps(c, nc, w, nw) ||
        (bias && overlaps(c, nc, bias, static_cast<size_t>(N) * 2)))
        return ATTN_ERR_ALIAS;
    const int sms = device_sms();
    if (sms < 1) return ATTN_ERR_DEVICE;
    const bool bf16 = dtype == ATTN_BF16;
    // 256-row tiles (a third less operand traffic, but an epilogue the next tile waits
    // for) pay off once a tile's products dwarf its epilogue: measured on B200, from
    // K = 8192 with the GELU epilogue (+9 % at 8192^3, -7 % at K = 4096) and from
    // K = 4096 without it (+3-9 %).  Flags 2 / 4 force the 128- / 256-row tiles.
    const bool wide = M > 128 && K >= (act == GEMM_ACT_GELU ? 8192 : 4096);
    const int mh = (flags & 2u) ? 1 : (flags & 4u) ? 2 : wide ? 2 : 1;
    const int BM = 128 * mh;
    CUtensorMap ta, tw;
    if (!encode_2d(&ta, a, K, M, BM, bf16) || !encode_2d(&tw, w, K, N, gemm::BN, bf16))
        return ATTN_ERR_TENSORMAP;
    gemm::Params p;
    p.c = c;
    p.bias = bias;
    p.M = M;
    p.N = N;
    p.K = K;
    p.num_m = (M + BM - 1) / BM;
    p.num_n = (N + gemm::BN - 1) / gemm::BN;
    p.num_k = (K + gemm::BK - 1) / gemm::BK;
    const int64_t tiles = static_cast<int64_t>(p.num_m) * p.num_n;
    if (tiles > INT_MAX) return ATTN_ERR_SHAPE;
    p.num_tiles = static_cast<int>(tiles);
    p.flags = flags & 1u;
    const int grid = p.num_tiles < sms ? p.num_tiles : sms;
    if (mh == 2)
        return bf16 ? launch_act<true, 2>(ta, tw, p, act, grid, stream)
                    : launch_act<false, 2>(ta, tw, p, act, grid, stream);
    return bf16 ? launch_act<true, 1>(ta, tw, p, act, grid, stream)
                : launch_act<false, 1>(ta, tw, p, act, grid, stream);
}

}  // namespace

// Read and clear this file's status word (attn_fwd_status reports it with the
// attention kernels' word).  Internal to the library.
__attribute__((visibility("hidden"))) int gemm_status_take(cudaStream_t s, int* out) {
    int v = 0;
    const int zero = 0;
    if (cudaMemcpyFromSymbolAsync(&v, gemm::g_gemm_status, sizeof(int), 0,
                                  cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaMemcpyToSymbolAsync(gemm::g_gemm_status, &zero, sizeof(int), 0,
                                cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_LAUNCH;
    }
    *out = v;
    return ATTN_OK;
}

extern "C" {

int gemm_bias_act(const void* a, const void* w, const void* bias, void* c, int M, int N, int K,
                  int act, int dtype, attn_stream_t stream) {
    return run(a, w, bias, c, M, N, K, act, dtype, reinterpret_cast<cudaStream_t>(stream), 0u);
}

int gemm_bias_act_debug(const void* a, const void* w, const void* bias, void* c, int M, int N,
                        int K, int act, int dtype, attn_stream_t stream, unsigned flags) {
    return run(a, w, bias, c, M, N, K, act, dtype, reinterpret_cast<cudaStream_t>(stream),
               flags & 7u);
}

}  // extern "C"
