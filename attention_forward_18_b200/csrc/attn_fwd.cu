// attn_fwd.cu -- host side of the C ABI declared in include/attn_fwd.h: argument
// checks, TMA descriptor encoding, kernel selection and launch.
#include <cuda.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "attn_fwd.h"
#include "attn_fwd_kernel.cuh"
#include "attn_fwd_wide_kernel.cuh"
#include "attn_fwd_pair_kernel.cuh"
#include "attn_merge.cuh"

// Library-owned scratch of attn_fwd_splitkv_noalloc: one copy per device, in the
// module's static device memory (no allocation by this library at call time).
static __device__ __align__(256) unsigned char g_noalloc_scratch[ATTN_SPLITKV_NOALLOC_SCRATCH_BYTES];

// Status word of the GEMM kernels (gemm_bias_act.cu): read and cleared on `s`.
int gemm_status_take(cudaStream_t s, int* out);

namespace {

constexpr int kMaxSeq = 1 << 24;
constexpr int kMaxHeads = 1 << 24;
constexpr int kMaxDevices = 64;
constexpr int kMaxSplits = 1024;

// cuTensorMapEncodeTiled, fetched through the runtime so the library needs no
// link against libcuda.
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

// [BH, S, D] 16-bit tensor seen as 3-D (D innermost); box = 64 elements (128 bytes,
// the swizzle span) x box_rows rows x 1 head; rows past S and columns past D read as
// zeros.
bool encode_qkv_map(CUtensorMap* m, const void* base, int D, int S, int BH, bool bf16,
                    int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S),
                                static_cast<cuuint64_t>(BH)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2,
                                   static_cast<cuuint64_t>(S) * D * 2};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(attn::CHUNK_ELEMS),
                               static_cast<cuuint32_t>(box_rows), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r =
        fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
           const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The same tensor seen as 4-D (cw columns, S rows, D/cw column chunks, BH heads): a box
// of cw columns x box_rows rows x box_chunks chunks lands in shared memory chunk-major,
// each chunk box_rows x (2 cw) bytes in the swizzle of that row size (cw = 64: 128-byte
// swizzle; cw = 32: 64-byte swizzle), as box_chunks 3-D boxes would.  D a multiple of cw.
bool encode_chunked_map(CUtensorMap* m, const void* base, int D, int S, int BH, bool bf16,
                        int box_rows, int box_chunks, int cw) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(cw), static_cast<cuuint64_t>(S),
                                static_cast<cuuint64_t>(D / cw), static_cast<cuuint64_t>(BH)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2,
                                   static_cast<cuuint64_t>(cw) * 2,
                                   static_cast<cuuint64_t>(S) * D * 2};
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(cw), static_cast<cuuint32_t>(box_rows),
                               static_cast<cuuint32_t>(box_chunks), 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r =
        fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4,
           const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
           cw == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Per-device facts checked once: compute capability 10.0 and the SM count (the
// persistent grid has one CTA per SM).  Kept for the life of the process (not valid
// across cudaDeviceReset, like the other per-device set-up below).
int check_device(int* num_sms) {
    static int dev_ok[kMaxDevices];  // 0 unknown, 1 ok, -1 not sm_100
    static int sms[kMaxDevices];
    static std::mutex mu;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return ATTN_ERR_DEVICE;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (dev_ok[dev] == 0) {
        int major = 0, minor = 0, count = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return ATTN_ERR_DEVICE;
        }
        // the library carries sm_100a code only, which no other 10.x part runs
        dev_ok[dev] = (major == 10 && minor == 0 && count > 0) ? 1 : -1;
        sms[dev] = count;
    }
    if (num_sms) *num_sms = sms[dev];
    return dev_ok[dev] == 1 ? ATTN_OK : ATTN_ERR_DEVICE;
}

// Device address of g_noalloc_scratch on the current device, looked up once per
// device (the first lookup may load the library's device code on that device).
int noalloc_scratch(void** out) {
    static void* ptr[kMaxDevices];
    static std::mutex mu;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return ATTN_ERR_DEVICE;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return ATTN_ERR_LAUNCH;
        }
        ptr[dev] = p;
    }
    *out = ptr[dev];
    return ATTN_OK;
}

// Head dimensions: 64 and 128 run at their size; 80, 96 and 112 run in the D = 128
// kernel with Q, K, V zero-padded by the TMA loads (columns past D read as zeros, so
// the scores and the output are unchanged) and O written for D columns.  192 and 256
// run in the wide kernel (one 128-row query tile per CTA, 64-key KV tiles).
bool head_dim_ok(int D) {
    return D == 64 || D == 80 || D == 96 || D == 112 || D == 128 || D == 192 || D == 256;
}
int kernel_d(int D) { return D <= 64 ? 64 : D <= 128 ? 128 : D; }
bool is_wide(int D) { return D > 128; }
// query rows per work unit, at the least over the kernels that can run D (the bound
// on the unit count checked by validate)
int unit_rows(int D) { return is_wide(D) ? attn::wide::WBM : attn::ROWS_PER_CTA; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

// Chunks of heads attn_fwd_host pipelines its copies over: at most 8, each at least
// 8 MB of Q, K and V (below that a copy's fixed cost outweighs the overlap), one for
// small passes.
int host_chunks(int BH, int Sq, int Sk, int D) {
    const int64_t in_bytes = static_cast<int64_t>(BH) * (Sq + 2 * static_cast<int64_t>(Sk)) * D * 2;
    int64_t n = in_bytes / (8ll << 20);
    if (n > 8) n = 8;
    if (n > BH) n = BH;
    if (n < 1) n = 1;
    const int per = static_cast<int>((BH + n - 1) / n);
    return (BH + per - 1) / per;
}

// attn_fwd_host's two copy streams (non-blocking) and the events that order them
// against the caller's stream: created once per device on first use and kept for the
// life of the process (not valid across cudaDeviceReset); `mu` keeps one call's
// records and waits together.
struct HostPipe {
    cudaStream_t in_stream = nullptr, out_stream = nullptr;
    cudaEvent_t start = nullptr, in = nullptr, out = nullptr, end = nullptr;
    std::mutex mu;
};

int host_pipe(HostPipe** out) {
    static HostPipe pipes[kMaxDevices];
    static int state[kMaxDevices];  // 0 not made, 1 ready, -1 failed
    static std::mutex mu;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return ATTN_ERR_DEVICE;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (state[dev] == 0) {
        HostPipe& p = pipes[dev];
        const unsigned ef = cudaEventDisableTiming;
        const bool made =
            cudaStreamCreateWithFlags(&p.in_stream, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&p.out_stream, cudaStreamNonBlocking) == cudaSuccess &&
            cudaEventCreateWithFlags(&p.start, ef) == cudaSuccess &&
            cudaEventCreateWithFlags(&p.in, ef) == cudaSuccess &&
            cudaEventCreateWithFlags(&p.out, ef) == cudaSuccess &&
            cudaEventCreateWithFlags(&p.end, ef) == cudaSuccess;
        if (!made) cudaGetLastError();
        state[dev] = made ? 1 : -1;
    }
    if (state[dev] != 1) return ATTN_ERR_LAUNCH;
    *out = &pipes[dev];
    return ATTN_OK;
}

// Hkv: heads of K and V (a divisor of H; H for plain multi-head attention).
int validate(const void* q, const void* k, const void* v, const void* o, const float* lse,
             int B, int H, int Hkv, int Sq, int Sk, int D, float scale, int dtype) {
    if (!q || !k || !v || !o) return ATTN_ERR_NULLPTR;
    if (dtype != ATTN_F16 && dtype != ATTN_BF16) return ATTN_ERR_DTYPE;
    if (!head_dim_ok(D)) return ATTN_ERR_HEADDIM;
    if (B < 1 || H < 1 || Hkv < 1 || Sq < 1 || Sk < 1 || H % Hkv != 0) return ATTN_ERR_SHAPE;
    if (Sq > kMaxSeq || Sk > kMaxSeq) return ATTN_ERR_SHAPE;
    const int64_t bh = static_cast<int64_t>(B) * H;
    if (bh > kMaxHeads) return ATTN_ERR_SHAPE;
    // the kernel's rows: g = H / Hkv query heads packed per K/V head
    const int64_t rows = static_cast<int64_t>(H / Hkv) * Sq;
    if (rows > kMaxSeq) return ATTN_ERR_SHAPE;
    const int64_t n_qp = (rows + unit_rows(D) - 1) / unit_rows(D);
    if (n_qp * B * Hkv > INT_MAX) return ATTN_ERR_SHAPE;
    if (!std::isfinite(scale)) return ATTN_ERR_SCALE;
    auto mis16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; };
    if (mis16(q) || mis16(k) || mis16(v) || mis16(o)) return ATTN_ERR_ALIGN;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return ATTN_ERR_ALIGN;
    const size_t nq = static_cast<size_t>(bh) * Sq * D * 2;
    const size_t nk = static_cast<size_t>(B) * Hkv * Sk * D * 2;
    if (overlaps(o, nq, q, nq) || overlaps(o, nq, k, nk) || overlaps(o, nq, v, nk))
        return ATTN_ERR_ALIAS;
    if (lse) {
        const size_t nl = static_cast<size_t>(bh) * Sq * 4;
        if (overlaps(lse, nl, q, nq) || overlaps(lse, nl, k, nk) || overlaps(lse, nl, v, nk) ||
            overlaps(lse, nl, o, nq))
            return ATTN_ERR_ALIAS;
    }
    return ATTN_OK;
}

template <int D, int NS, bool BF16, bool CAUSAL, bool NEG, bool SPLIT, bool GEN, bool DEC>
int launch_one(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
               const attn::Params& p, int grid, cudaStream_t stream) {
    auto kern = attn::attn_fwd_kernel<D, NS, BF16, CAUSAL, NEG, SPLIT, GEN, DEC>;
    constexpr int smem = attn::SmemLayout<D, NS>::ALLOC;
    static bool attr_set[kMaxDevices];
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_LAUNCH;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!attr_set[dev]) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
                cudaSuccess) {
                cudaGetLastError();
                return ATTN_ERR_LAUNCH;
            }
            attr_set[dev] = true;
        }
    }
    kern<<<grid, attn::NUM_THREADS, smem, stream>>>(tq, tk, tv, p);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

// Ring depth: as many K/V stages as fit beside the two Q tiles in shared memory.
template <int D>
constexpr int kStages = (D == 64) ? 5 : 2;

// Negative scales run their own instantiation (scores negated as they are read), so
// the common case carries no per-element sign handling.  The general causal forms
// (an offset or grouped heads) run their own instantiations too, so plain top-left
// causal attention keeps the simplest per-row arithmetic.
//
// Rows that all fit in query tile 0 (at most 128 packed query rows: decoding) take the
// DEC instantiations, where both softmax warpgroups work on that tile, on alternate KV
// tiles.  (Plain top-left causal attention with so few rows sees at most 128 keys, one
// KV tile: nothing to share, so it has no DEC instantiation.)
template <int D, bool BF16, bool SPLIT, bool CAUSAL, bool GEN>
int launch_neg_dec(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                   const attn::Params& p, int grid, cudaStream_t s) {
    constexpr int NS = kStages<D>;
    const bool neg = p.scale_log2 < 0.f;
    const bool dec = p.Sq <= attn::BM;
    if (dec && (!CAUSAL || GEN))
        return neg ? launch_one<D, NS, BF16, CAUSAL, true, SPLIT, GEN, !CAUSAL || GEN>(tq, tk, tv, p, grid, s)
                   : launch_one<D, NS, BF16, CAUSAL, false, SPLIT, GEN, !CAUSAL || GEN>(tq, tk, tv, p, grid, s);
    return neg ? launch_one<D, NS, BF16, CAUSAL, true, SPLIT, GEN, false>(tq, tk, tv, p, grid, s)
               : launch_one<D, NS, BF16, CAUSAL, false, SPLIT, GEN, false>(tq, tk, tv, p, grid, s);
}

template <int D, bool BF16, bool SPLIT>
int launch_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
             const attn::Params& p, int grid, bool causal, cudaStream_t s) {
    if (causal && (p.causal_off != 0 || p.sq_head != p.Sq))
        return launch_neg_dec<D, BF16, SPLIT, true, true>(tq, tk, tv, p, grid, s);
    if (causal) return launch_neg_dec<D, BF16, SPLIT, true, false>(tq, tk, tv, p, grid, s);
    return launch_neg_dec<D, BF16, SPLIT, false, false>(tq, tk, tv, p, grid, s);
}

template <bool SPLIT>
int launch_any(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
               const attn::Params& p, int grid, int D, bool bf16, bool causal,
               cudaStream_t s) {
    if (D == 64) return bf16 ? launch_d<64, true, SPLIT>(tq, tk, tv, p, grid, causal, s)
                             : launch_d<64, false, SPLIT>(tq, tk, tv, p, grid, causal, s);
    return bf16 ? launch_d<128, true, SPLIT>(tq, tk, tv, p, grid, causal, s)
                : launch_d<128, false, SPLIT>(tq, tk, tv, p, grid, causal, s);
}

template <int D, int NS, bool BF16, bool CAUSAL, bool NEG, bool SPLIT, bool GEN>
int launch_wide_one(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                    const attn::Params& p, int grid, cudaStream_t stream) {
    auto kern = attn::wide::attn_fwd_wide_kernel<D, NS, BF16, CAUSAL, NEG, SPLIT, GEN>;
    constexpr int smem = attn::wide::Layout<D, NS>::ALLOC;
    static bool attr_set[kMaxDevices];
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_LAUNCH;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!attr_set[dev]) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
                cudaSuccess) {
                cudaGetLastError();
                return ATTN_ERR_LAUNCH;
            }
            attr_set[dev] = true;
        }
    }
    kern<<<grid, attn::wide::NUM_THREADS, smem, stream>>>(tq, tk, tv, p);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

// D = 192 / 256 on CTA pairs: clusters of two CTAs, the grid sized to the clusters that
// can be resident at once (a persistent grid; the pair walks its units).
template <int PD, bool BF16, bool CAUSAL, bool NEG, bool SPLIT, bool GEN>
int launch_pair_one(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                    const attn::Params& p, int64_t n_units, cudaStream_t stream) {
    // K / V ring stages: D = 256 3 + 2 (224 KB with Q), D = 192 3 + 3 (192 KB)
    constexpr int NSK = 3, NSV = PD == 256 ? 2 : 3;
    auto kern = attn::pair::attn_fwd_pair_kernel<PD, NSK, NSV, BF16, CAUSAL, NEG, SPLIT, GEN>;
    constexpr int smem = attn::pair::Layout<PD, NSK, NSV>::ALLOC;
    static int max_clusters[kMaxDevices];  // 0: not yet known
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_LAUNCH;
    int clusters = 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (max_clusters[dev] == 0) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
                cudaSuccess) {
                cudaGetLastError();
                return ATTN_ERR_LAUNCH;
            }
            int sms = 0;
            if (check_device(&sms) != ATTN_OK) return ATTN_ERR_DEVICE;
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(static_cast<unsigned>(sms - sms % 2), 1, 1);
            cfg.blockDim = dim3(attn::pair::NUM_THREADS, 1, 1);
            cfg.dynamicSmemBytes = smem;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
                cudaGetLastError();
                return ATTN_ERR_LAUNCH;
            }
            max_clusters[dev] = n;
        }
        clusters = max_clusters[dev];
    }
    if (n_units < clusters) clusters = static_cast<int>(n_units);
    kern<<<2 * clusters, attn::pair::NUM_THREADS, smem, stream>>>(tq, tk, tv, p);
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

template <int PD, bool BF16, bool SPLIT>
int launch_pair_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                  const attn::Params& p, int64_t n_units, bool causal, cudaStream_t s) {
    const bool neg = p.scale_log2 < 0.f;
    if (causal && (p.causal_off != 0 || p.sq_head != p.Sq))
        return neg ? launch_pair_one<PD, BF16, true, true, SPLIT, true>(tq, tk, tv, p, n_units, s)
                   : launch_pair_one<PD, BF16, true, false, SPLIT, true>(tq, tk, tv, p, n_units, s);
    if (causal)
        return neg ? launch_pair_one<PD, BF16, true, true, SPLIT, false>(tq, tk, tv, p, n_units, s)
                   : launch_pair_one<PD, BF16, true, false, SPLIT, false>(tq, tk, tv, p, n_units, s);
    return neg ? launch_pair_one<PD, BF16, false, true, SPLIT, false>(tq, tk, tv, p, n_units, s)
               : launch_pair_one<PD, BF16, false, false, SPLIT, false>(tq, tk, tv, p, n_units, s);
}

template <bool SPLIT>
int launch_pair(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                const attn::Params& p, int64_t n_units, int D, bool bf16, bool causal,
                cudaStream_t s) {
    if (D == 192) return bf16 ? launch_pair_d<192, true, SPLIT>(tq, tk, tv, p, n_units, causal, s)
                              : launch_pair_d<192, false, SPLIT>(tq, tk, tv, p, n_units, causal, s);
    return bf16 ? launch_pair_d<256, true, SPLIT>(tq, tk, tv, p, n_units, causal, s)
                : launch_pair_d<256, false, SPLIT>(tq, tk, tv, p, n_units, causal, s);
}

// Wide kernel ring depth: 64-key K/V stages beside the 128-row Q tile (~192 KB).
template <int D>
constexpr int kWideStages = (D == 256) ? 2 : 3;

template <int D, bool BF16, bool SPLIT>
int launch_wide_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                  const attn::Params& p, int grid, bool causal, cudaStream_t s) {
    constexpr int NS = kWideStages<D>;
    const bool neg = p.scale_log2 < 0.f;
    if (causal && (p.causal_off != 0 || p.sq_head != p.Sq))
        return neg ? launch_wide_one<D, NS, BF16, true, true, SPLIT, true>(tq, tk, tv, p, grid, s)
                   : launch_wide_one<D, NS, BF16, true, false, SPLIT, true>(tq, tk, tv, p, grid, s);
    if (causal)
        return neg ? launch_wide_one<D, NS, BF16, true, true, SPLIT, false>(tq, tk, tv, p, grid, s)
                   : launch_wide_one<D, NS, BF16, true, false, SPLIT, false>(tq, tk, tv, p, grid, s);
    return neg ? launch_wide_one<D, NS, BF16, false, true, SPLIT, false>(tq, tk, tv, p, grid, s)
               : launch_wide_one<D, NS, BF16, false, false, SPLIT, false>(tq, tk, tv, p, grid, s);
}

template <bool SPLIT>
int launch_wide(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                const attn::Params& p, int grid, int D, bool bf16, bool causal,
                cudaStream_t s) {
    if (D == 192) return bf16 ? launch_wide_d<192, true, SPLIT>(tq, tk, tv, p, grid, causal, s)
                              : launch_wide_d<192, false, SPLIT>(tq, tk, tv, p, grid, causal, s);
    return bf16 ? launch_wide_d<256, true, SPLIT>(tq, tk, tv, p, grid, causal, s)
                : launch_wide_d<256, false, SPLIT>(tq, tk, tv, p, grid, causal, s);
}

// Workspace of a split pass: partial O [n_splits, B*H, Sq, D] fp32, then partial LSE
// [n_splits, B*H, Sq] fp32 at the next 256-byte boundary.
size_t ws_o_bytes(int B, int H, int Sq, int D, int n_splits) {
    const size_t b = static_cast<size_t>(n_splits) * B * H * Sq * D * 4;
    return (b + 255) & ~static_cast<size_t>(255);
}
size_t ws_bytes(int B, int H, int Sq, int D, int n_splits) {
    return ws_o_bytes(B, H, Sq, D, n_splits) + static_cast<size_t>(n_splits) * B * H * Sq * 4;
}

int launch_merge(const float* ws_o, const float* ws_lse, void* o, float* lse, int n_splits,
                 int64_t rows, int D, bool bf16, cudaStream_t s) {
    const int64_t threads = rows * 32;
    const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
    if (D == 64) {
        if (bf16) attn::attn_splitkv_merge_kernel<64, true><<<blocks, 256, 0, s>>>(ws_o, ws_lse, o, lse, n_splits, rows);
        else attn::attn_splitkv_merge_kernel<64, false><<<blocks, 256, 0, s>>>(ws_o, ws_lse, o, lse, n_splits, rows);
    } else if (D == 192) {
        if (bf16) attn::attn_splitkv_merge_kernel<192, true><<<blocks, 256, 0, s>>>(ws_o, ws_lse, o, lse, n_splits, rows);
        else attn::attn_splitkv_merge_kernel<192, false><<<blocks, 256, 0, s>>>(ws_o, ws_lse, o, lse, n_splits, rows);
    } else if (D == 256) {
        if (bf16) attn::attn_splitkv_merge_kernel<256, true><<<blocks, 256, 0, s>>>(ws_o, ws_lse, o, lse, n_splits, rows);
        else attn::attn_splitkv_merge_kernel<256, false><<<blocks, 256, 0, s>>>(ws_o, ws_lse, o, lse, n_splits, rows);
    } else if (D != 128) {
        if (bf16) attn::attn_splitkv_merge_any_d<true><<<blocks, 256, 0, s>>>(ws_o, ws_lse, o, lse, n_splits, rows, D);
        else attn::attn_splitkv_merge_any_d<false><<<blocks, 256, 0, s>>>(ws_o, ws_lse, o, lse, n_splits, rows, D);
    } else {
        if (bf16) attn::attn_splitkv_merge_kernel<128, true><<<blocks, 256, 0, s>>>(ws_o, ws_lse, o, lse, n_splits, rows);
        else attn::attn_splitkv_merge_kernel<128, false><<<blocks, 256, 0, s>>>(ws_o, ws_lse, o, lse, n_splits, rows);
    }
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

// n_splits == 0: the whole pass (16-bit O and LSE written by the attention kernel);
// n_splits >= 1: a split pass through `workspace`, then the merge kernel.
// Hkv: K/V heads (divides H); mask: ATTN_MASK_*.
// Host-side debug flag of attn_fwd_debug: report a failed TMA descriptor encoding.
constexpr unsigned kFlagFailTensorMap = 2u;

int run(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv,
        int Sq, int Sk, int D, int mask, float scale, int dtype, cudaStream_t stream,
        unsigned flags, int n_splits = 0, void* workspace = nullptr, size_t workspace_bytes = 0) {
    int rc = validate(q, k, v, o, lse, B, H, Hkv, Sq, Sk, D, scale, dtype);
    if (rc != ATTN_OK) return rc;
    if (mask != ATTN_MASK_NONE && mask != ATTN_MASK_CAUSAL &&
        mask != ATTN_MASK_CAUSAL_BOTTOM_RIGHT)
        return ATTN_ERR_MASK;
    if (n_splits < 0 || n_splits > kMaxSplits) return ATTN_ERR_SHAPE;
    if (n_splits > 0) {
        // the merge kernel runs one warp per (head, query row) in a 1-D grid
        if (static_cast<int64_t>(B) * H * Sq > static_cast<int64_t>(INT_MAX) * 8)
            return ATTN_ERR_SHAPE;
        if (!workspace) return ATTN_ERR_NULLPTR;
        if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_ALIGN;
        const size_t need = ws_bytes(B, H, Sq, D, n_splits);
        if (workspace_bytes < need) return ATTN_ERR_WORKSPACE;
        const size_t nq = static_cast<size_t>(B) * H * Sq * D * 2;
        const size_t nk = static_cast<size_t>(B) * Hkv * Sk * D * 2;
        if (overlaps(workspace, need, q, nq) || overlaps(workspace, need, k, nk) ||
            overlaps(workspace, need, v, nk) || overlaps(workspace, need, o, nq) ||
            (lse && overlaps(workspace, need, lse, static_cast<size_t>(B) * H * Sq * 4)))
            return ATTN_ERR_ALIAS;
    }
    int num_sms = 0;
    if ((rc = check_device(&num_sms)) != ATTN_OK) return rc;

    // The kernel's view: B*Hkv heads of g*Sq query rows (the g query heads of a K/V
    // head are adjacent in [B, H, Sq, D]), Sk keys.
    const int BH = B * Hkv;
    const int rows = (H / Hkv) * Sq;
    const bool bf16 = dtype == ATTN_BF16;
    // D = 192 / 256 with more than one query tile of packed rows run on CTA pairs (the
    // D <= 128 geometry: 256-row units, 128-key tiles, each CTA holding half of every
    // K and V tile); with fewer rows (decoding) they run in the wide kernel.
    const bool pair_path = is_wide(D) && rows > attn::BM;
    const bool wide = is_wide(D) && !pair_path;
    const int kv_keys = wide ? attn::wide::WBN : attn::BN;
    const int q_units = wide ? attn::wide::WBM : attn::ROWS_PER_CTA;
    CUtensorMap tq, tk, tv;
    if (flags & kFlagFailTensorMap) return ATTN_ERR_TENSORMAP;
    if (pair_path) {
        // one box per half tile: Q 128 rows and K 64 keys, all 64-column chunks; V 128
        // keys, this CTA's D/2 columns (64-column chunks at D = 256, 32-column at 192)
        const int vcw = D == 256 ? 64 : 32;
        const int nch = D / attn::CHUNK_ELEMS;
        if (!encode_chunked_map(&tq, q, D, rows, BH, bf16, attn::BM, nch, attn::CHUNK_ELEMS) ||
            !encode_chunked_map(&tk, k, D, Sk, BH, bf16, 64, nch, attn::CHUNK_ELEMS) ||
            !encode_chunked_map(&tv, v, D, Sk, BH, bf16, attn::BN, D / 2 / vcw, vcw))
            return ATTN_ERR_TENSORMAP;
    } else if (!encode_qkv_map(&tq, q, D, rows, BH, bf16, attn::BM) ||
               !encode_qkv_map(&tk, k, D, Sk, BH, bf16, wide ? 64 : attn::BN) ||
               !encode_qkv_map(&tv, v, D, Sk, BH, bf16, wide ? 64 : attn::BN)) {
        return ATTN_ERR_TENSORMAP;
    }

    attn::Params p;
    p.o = o;
    p.lse = lse;
    p.Sq = rows;
    p.Sk = Sk;
    p.BH = BH;
    p.n_qp = (rows + q_units - 1) / q_units;  // query units (wide: single tiles)
    p.sq_head = Sq;
    p.d_out = D;
    p.causal_off = mask == ATTN_MASK_CAUSAL_BOTTOM_RIGHT ? Sk - Sq : 0;
    const int n_kv = (Sk + kv_keys - 1) / kv_keys;
    p.n_splits = n_splits > 0 ? n_splits : 1;
    p.chunk_tiles = (n_kv + p.n_splits - 1) / p.n_splits;

    p.ws_o = n_splits > 0 ? static_cast<float*>(workspace) : nullptr;
    p.ws_lse = n_splits > 0 ? reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                                       ws_o_bytes(B, H, Sq, D, n_splits))
                            : nullptr;
    p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634074);
    // A zero scale gives uniform weights over the visible keys; the kernel needs a
    // nonzero multiplier to keep masked scores at -inf (not -inf * 0 = NaN), and with
    // 1e-30 every visible weight is 2^(~1e-28) = 1.0f exactly.
    if (p.scale_log2 == 0.f) p.scale_log2 = 1e-30f;
    p.flags = flags & attn::FLAG_SKIP_Q_LOAD;
    // persistent: one CTA per SM (at most one per work unit), each walking its units
    const int64_t n_units = static_cast<int64_t>(p.n_qp) * BH * p.n_splits;
    if (n_units > INT_MAX) return ATTN_ERR_SHAPE;
    const int grid = n_units < num_sms ? static_cast<int>(n_units) : num_sms;
    const bool c = mask != ATTN_MASK_NONE;
    if (n_splits == 0) {
        if (pair_path) return launch_pair<false>(tq, tk, tv, p, n_units, D, bf16, c, stream);
        return wide ? launch_wide<false>(tq, tk, tv, p, grid, D, bf16, c, stream)
                    : launch_any<false>(tq, tk, tv, p, grid, kernel_d(D), bf16, c, stream);
    }
    if (pair_path)
        rc = launch_pair<true>(tq, tk, tv, p, n_units, D, bf16, c, stream);
    else
        rc = wide ? launch_wide<true>(tq, tk, tv, p, grid, D, bf16, c, stream)
                  : launch_any<true>(tq, tk, tv, p, grid, kernel_d(D), bf16, c, stream);
    if (rc != ATTN_OK) return rc;
    return launch_merge(p.ws_o, p.ws_lse, o, lse, n_splits, static_cast<int64_t>(B) * H * Sq, D,
                        bf16, stream);
}

int mask_of(int causal) { return causal ? ATTN_MASK_CAUSAL : ATTN_MASK_NONE; }

// Split count for `units` (query block, head) pairs over KV tiles 0..n_kv-1 on `slots`
// units that run at once (SMs, or CTA pairs): persistent CTAs take units round-robin,
// so a pass lasts about
//   ceil(units * n / slots) rounds x (tiles per range + a fill of `fill` tiles)
// (the fill of a range, ~2 tiles of 128 keys, is ~4 of the wide kernel's 64-key tiles);
// the n with the least of that (the fewest splits among equals: less to merge).
int balanced_splits(int64_t units, int n_kv, int slots, int fill) {
    const int num_sms = slots;
    int best = 1;
    int64_t best_cost = INT64_MAX;
    const int n_hi = n_kv < kMaxSplits ? n_kv : kMaxSplits;
    for (int n = 1; n <= n_hi; ++n) {
        const int chunk = (n_kv + n - 1) / n;
        if ((n_kv + chunk - 1) / chunk != n) continue;  // some range would be empty
        const int64_t rounds = (units * n + num_sms - 1) / num_sms;
        const int64_t cost = rounds * (chunk + fill);
        if (cost < best_cost) {
            best_cost = cost;
            best = n;
        }
    }
    return best;
}

}  // namespace

extern "C" {

int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
             int Sq, int Sk, int D, int causal, float scale, int dtype, attn_stream_t stream) {
    return run(q, k, v, o, lse, B, H, H, Sq, Sk, D, mask_of(causal), scale, dtype,
               reinterpret_cast<cudaStream_t>(stream), 0u);
}

int attn_fwd_debug(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                   int H, int Sq, int Sk, int D, int causal, float scale, int dtype,
                   attn_stream_t stream, unsigned flags) {
    return run(q, k, v, o, lse, B, H, H, Sq, Sk, D, mask_of(causal), scale, dtype,
               reinterpret_cast<cudaStream_t>(stream),
               flags & (attn::FLAG_SKIP_Q_LOAD | kFlagFailTensorMap));
}

int attn_fwd_host(const void* q_host, const void* k_host, const void* v_host, void* o_host,
                  float* lse_host, void* q_dev, void* k_dev, void* v_dev, void* o_dev,
                  float* lse_dev, int B, int H, int Sq, int Sk, int D, int causal, float scale,
                  int dtype, attn_stream_t stream) {
    if (!q_host || !k_host || !v_host || !o_host) return ATTN_ERR_NULLPTR;
    int rc = validate(q_dev, k_dev, v_dev, o_dev, lse_dev, B, H, H, Sq, Sk, D, scale, dtype);
    if (rc != ATTN_OK) return rc;
    if ((rc = check_device(nullptr)) != ATTN_OK) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int BH = B * H;
    const bool lse_out = lse_host && lse_dev;
    const int n = host_chunks(BH, Sq, Sk, D);
    const int per = (BH + n - 1) / n;
    // heads [h0, h0 + nh) of the flattened [B*H] axis: contiguous in every tensor
    auto h2d = [&](int h0, int nh, cudaStream_t st) {
        const size_t oq = static_cast<size_t>(h0) * Sq * D * 2, ok = static_cast<size_t>(h0) * Sk * D * 2;
        const size_t nq = static_cast<size_t>(nh) * Sq * D * 2, nk = static_cast<size_t>(nh) * Sk * D * 2;
        return cudaMemcpyAsync(static_cast<char*>(q_dev) + oq, static_cast<const char*>(q_host) + oq,
                               nq, cudaMemcpyHostToDevice, st) == cudaSuccess &&
               cudaMemcpyAsync(static_cast<char*>(k_dev) + ok, static_cast<const char*>(k_host) + ok,
                               nk, cudaMemcpyHostToDevice, st) == cudaSuccess &&
               cudaMemcpyAsync(static_cast<char*>(v_dev) + ok, static_cast<const char*>(v_host) + ok,
                               nk, cudaMemcpyHostToDevice, st) == cudaSuccess;
    };
    auto d2h = [&](int h0, int nh, cudaStream_t st) {
        const size_t oq = static_cast<size_t>(h0) * Sq * D * 2, nq = static_cast<size_t>(nh) * Sq * D * 2;
        const size_t ol = static_cast<size_t>(h0) * Sq, nl = static_cast<size_t>(nh) * Sq * 4;
        return cudaMemcpyAsync(static_cast<char*>(o_host) + oq, static_cast<const char*>(o_dev) + oq,
                               nq, cudaMemcpyDeviceToHost, st) == cudaSuccess &&
               (!lse_out || cudaMemcpyAsync(lse_host + ol, lse_dev + ol, nl,
                                            cudaMemcpyDeviceToHost, st) == cudaSuccess);
    };
    auto pass = [&](int h0, int nh) {
        const size_t oq = static_cast<size_t>(h0) * Sq * D * 2, ok = static_cast<size_t>(h0) * Sk * D * 2;
        return run(static_cast<const char*>(q_dev) + oq, static_cast<const char*>(k_dev) + ok,
                   static_cast<const char*>(v_dev) + ok, static_cast<char*>(o_dev) + oq,
                   lse_dev ? lse_dev + static_cast<size_t>(h0) * Sq : nullptr, 1, nh, nh, Sq,
                   Sk, D, mask_of(causal), scale, dtype, s, 0u);
    };
    if (n == 1) {
        if (!h2d(0, BH, s)) {
            cudaGetLastError();
            return ATTN_ERR_LAUNCH;
        }
        if ((rc = pass(0, BH)) != ATTN_OK) return rc;
        if (!d2h(0, BH, s)) {
            cudaGetLastError();
            return ATTN_ERR_LAUNCH;
        }
        return ATTN_OK;
    }
    // Head chunks in a three-stage pipeline: chunk c+1's inputs cross the host link on
    // one copy stream while chunk c's pass runs on `stream` and chunk c-1's outputs
    // return on another, so the two directions of the link and the kernel overlap.
    HostPipe* hp = nullptr;
    if ((rc = host_pipe(&hp)) != ATTN_OK) return rc;
    std::lock_guard<std::mutex> lock(hp->mu);
    bool ok = cudaEventRecord(hp->start, s) == cudaSuccess &&
              cudaStreamWaitEvent(hp->in_stream, hp->start, 0) == cudaSuccess &&
              cudaStreamWaitEvent(hp->out_stream, hp->start, 0) == cudaSuccess;
    for (int h0 = 0; ok && h0 < BH; h0 += per) {
        const int nh = BH - h0 < per ? BH - h0 : per;
        ok = h2d(h0, nh, hp->in_stream) && cudaEventRecord(hp->in, hp->in_stream) == cudaSuccess &&
             cudaStreamWaitEvent(s, hp->in, 0) == cudaSuccess;
        if (ok && (rc = pass(h0, nh)) != ATTN_OK) break;
        ok = ok && cudaEventRecord(hp->out, s) == cudaSuccess &&
             cudaStreamWaitEvent(hp->out_stream, hp->out, 0) == cudaSuccess &&
             d2h(h0, nh, hp->out_stream);
    }
    // both copy streams rejoin `stream` on every path, so that the caller's stream
    // orders everything this call queued (and a capture into a graph stays joined)
    const bool joined = cudaEventRecord(hp->in, hp->in_stream) == cudaSuccess &&
                        cudaStreamWaitEvent(s, hp->in, 0) == cudaSuccess &&
                        cudaEventRecord(hp->end, hp->out_stream) == cudaSuccess &&
                        cudaStreamWaitEvent(s, hp->end, 0) == cudaSuccess;
    if (rc != ATTN_OK) return rc;
    if (!ok || !joined) {
        cudaGetLastError();
        return ATTN_ERR_LAUNCH;
    }
    return ATTN_OK;
}

size_t attn_fwd_splitkv_workspace_bytes(int B, int H, int Sq, int D, int n_splits) {
    if (B < 1 || H < 1 || Sq < 1 || !head_dim_ok(D) || n_splits < 1 ||
        n_splits > kMaxSplits)
        return 0;
    return ws_bytes(B, H, Sq, D, n_splits);
}

int attn_fwd_splitkv_default_splits(int B, int H, int Sq, int Sk, int D, int causal) {
    return attn_fwd_ex_default_splits(B, H, H, Sq, Sk, D, mask_of(causal));
}

int attn_fwd_ex_default_splits(int B, int H, int H_kv, int Sq, int Sk, int D, int mask) {
    if (B < 1 || H < 1 || H_kv < 1 || H % H_kv != 0 || Sq < 1 || Sk < 1 || !head_dim_ok(D) ||
        mask < 0 || mask > ATTN_MASK_CAUSAL_BOTTOM_RIGHT)
        return 0;
    int num_sms = 0;
    if (check_device(&num_sms) != ATTN_OK) num_sms = 148;
    // the geometry of the kernel run() picks for these sizes: D <= 128 and the CTA pairs
    // take 256-row units and 128-key tiles (a pair's unit on two SMs); the wide kernel
    // (D = 192 / 256, at most 128 packed rows) 128-row units and 64-key tiles
    const int64_t rows = static_cast<int64_t>(H / H_kv) * Sq;
    const bool wide = is_wide(D) && rows <= attn::BM;
    const bool pair = is_wide(D) && !wide;
    const int q_units = wide ? attn::wide::WBM : attn::ROWS_PER_CTA;
    const int kv_keys = wide ? attn::wide::WBN : attn::BN;
    const int64_t units = (rows + q_units - 1) / q_units * B * H_kv;
    // with the top-left causal mask no row sees a key past min(Sq, Sk)
    const int keys = mask == ATTN_MASK_CAUSAL ? (Sq < Sk ? Sq : Sk) : Sk;
    return balanced_splits(units, (keys + kv_keys - 1) / kv_keys, pair ? num_sms / 2 : num_sms,
                           2 * attn::BN / kv_keys);
}

int attn_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int H, int Sq, int Sk, int D, int causal, float scale, int dtype,
                     int n_splits, void* workspace, size_t workspace_bytes,
                     attn_stream_t stream) {
    if (n_splits < 1) return ATTN_ERR_SHAPE;
    return run(q, k, v, o, lse, B, H, H, Sq, Sk, D, mask_of(causal), scale, dtype,
               reinterpret_cast<cudaStream_t>(stream), 0u, n_splits, workspace, workspace_bytes);
}

int attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                int H_kv, int Sq, int Sk, int D, int mask, float scale, int dtype, int n_splits,
                void* workspace, size_t workspace_bytes, attn_stream_t stream) {
    return run(q, k, v, o, lse, B, H, H_kv, Sq, Sk, D, mask, scale, dtype,
               reinterpret_cast<cudaStream_t>(stream), 0u, n_splits, workspace, workspace_bytes);
}

int attn_fwd_splitkv_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                             int B, int H, int Sq, int Sk, int D, int causal, float scale,
                             int dtype, int n_splits, attn_stream_t stream) {
    int rc = validate(q, k, v, o, lse, B, H, H, Sq, Sk, D, scale, dtype);
    if (rc != ATTN_OK) return rc;
    if (n_splits < 1 || n_splits > kMaxSplits) return ATTN_ERR_SHAPE;
    if (ws_bytes(B, H, Sq, D, n_splits) > ATTN_SPLITKV_NOALLOC_SCRATCH_BYTES)
        return ATTN_ERR_WORKSPACE;
    if ((rc = check_device(nullptr)) != ATTN_OK) return rc;
    void* scratch = nullptr;
    if ((rc = noalloc_scratch(&scratch)) != ATTN_OK) return rc;
    return run(q, k, v, o, lse, B, H, H, Sq, Sk, D, mask_of(causal), scale, dtype,
               reinterpret_cast<cudaStream_t>(stream), 0u, n_splits, scratch,
               ATTN_SPLITKV_NOALLOC_SCRATCH_BYTES);
}

int attn_fwd_status(attn_stream_t stream, int* device_status) {
    if (!device_status) return ATTN_ERR_NULLPTR;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int value = 0;
    const int zero = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess ||
        cudaMemcpyFromSymbolAsync(&value, attn::g_attn_status, sizeof(int), 0,
                                  cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaMemcpyToSymbolAsync(attn::g_attn_status, &zero, sizeof(int), 0,
                                cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_LAUNCH;
    }
    // the GEMM kernels keep their own word (another translation unit)
    int gemm_value = 0;
    if (gemm_status_take(s, &gemm_value) != ATTN_OK) return ATTN_ERR_LAUNCH;
    *device_status = value != 0 ? value : gemm_value;
    return ATTN_OK;
}

const char* attn_fwd_strerror(int code) {
    switch (code) {
        case ATTN_OK: return "ok";
        case ATTN_ERR_NULLPTR: return "null pointer argument";
        case ATTN_ERR_ALIGN: return "misaligned pointer (q/k/v/o need 16 bytes, lse 4)";
        case ATTN_ERR_SHAPE: return "bad shape (B, H, Sq, Sk >= 1 and within limits)";
        case ATTN_ERR_HEADDIM: return "unsupported head dimension (64, 80, 96, 112, 128, 192 or 256)";
        case ATTN_ERR_DTYPE: return "unsupported dtype (ATTN_F16 or ATTN_BF16)";
        case ATTN_ERR_TENSORMAP: return "TMA descriptor encoding failed";
        case ATTN_ERR_LAUNCH: return "CUDA call or kernel launch failed";
        case ATTN_ERR_TIMEOUT: return "kernel pipeline wait timed out";
        case ATTN_ERR_SCALE: return "scale is not finite";
        case ATTN_ERR_ALIAS: return "output overlaps an input";
        case ATTN_ERR_DEVICE: return "no usable sm_100 CUDA device";
        case ATTN_ERR_MASK: return "mask is not one of ATTN_MASK_*";
        case ATTN_ERR_WORKSPACE: return "workspace smaller than attn_fwd_splitkv_workspace_bytes";
        default: return "unknown error code";
    }
}

int attn_fwd_abi_version(void) { return 2; }

}  // extern "C"
