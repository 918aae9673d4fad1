// row_softmax.cu -- the standalone row-wise softmax of the C ABI in
// include/row_softmax.h:  y[r, :] = exp(x[r, :] - max_r) / sum exp(x[r, :] - max_r).
//
// Bound by HBM (a 16-bit element is read once and written once; a few flops each), so
// the design is about bytes in flight and coalescing, not arithmetic:
//   * rows of up to 8 KB: one warp per row; every lane issues all of its 16-byte loads
//     before any use, so a warp keeps a whole row in flight (64 warps per SM: up to
//     512 KB per SM in flight);
//   * rows of up to 128 KB: one CTA per row, the row again held in registers
//     (16-byte chunks, up to 8 per thread), max and sum reduced across the CTA;
//   * longer rows (or rows whose length breaks 16-byte alignment): a cluster of up to
//     8 CTAs per row, each CTA a contiguous slice, in two passes: an online max / sum
//     of the slice, an exchange of the CTAs' (max, sum) pairs through distributed
//     shared memory, then the normalised output (four 16-byte loads in flight per
//     thread in each pass).  The slice is read twice.
// Grids are persistent: (resident CTAs per SM) x (SMs), each group walking rows.
// exp is ex2 on d = x - max (the difference first, so |d| carries the only rounding),
// the sum accumulates in fp32 and the output is rounded once.
#include <cuda_runtime.h>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <climits>
#include <cstdint>
#include <mutex>

#include "attn_fwd.h"
#include "ptx.cuh"
#include "row_softmax.h"

namespace {

constexpr float kLog2e = 1.4426950408889634074f;

// ---------------------------------------------------------------- element access
template <int DT> struct Elem;
template <> struct Elem<ATTN_F16> {
    static constexpr int kBytes = 2;
    __device__ static float get(const void* p, int64_t i) {
        return __half2float(reinterpret_cast<const __half*>(p)[i]);
    }
    __device__ static void put(void* p, int64_t i, float v) {
        reinterpret_cast<__half*>(p)[i] = __float2half_rn(v);
    }
};
template <> struct Elem<ATTN_BF16> {
    static constexpr int kBytes = 2;
    __device__ static float get(const void* p, int64_t i) {
        return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
    }
    __device__ static void put(void* p, int64_t i, float v) {
        reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
    }
};
template <> struct Elem<SOFTMAX_F32> {
    static constexpr int kBytes = 4;
    __device__ static float get(const void* p, int64_t i) {
        return reinterpret_cast<const float*>(p)[i];
    }
    __device__ static void put(void* p, int64_t i, float v) {
        reinterpret_cast<float*>(p)[i] = v;
    }
};

// A 16-byte chunk as EPV floats (8 16-bit values or 4 fp32).
template <int DT> struct Chunk {
    static constexpr int EPV = 16 / Elem<DT>::kBytes;
    __device__ static void unpack(const uint4& c, float (&v)[EPV]) {
        const uint32_t w[4] = {c.x, c.y, c.z, c.w};
        if constexpr (DT == SOFTMAX_F32) {
#pragma unroll
            for (int e = 0; e < 4; ++e) v[e] = __uint_as_float(w[e]);
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if constexpr (DT == ATTN_F16) {
                    const __half2 h = *reinterpret_cast<const __half2*>(&w[e]);
                    const float2 f = __half22float2(h);
                    v[2 * e] = f.x;
                    v[2 * e + 1] = f.y;
                } else {
                    // bf16 -> fp32 is a 16-bit shift
                    v[2 * e] = __uint_as_float(w[e] << 16);
                    v[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
                }
            }
        }
    }
    __device__ static uint4 pack(const float (&v)[EPV]) {
        uint32_t w[4];
        if constexpr (DT == SOFTMAX_F32) {
#pragma unroll
            for (int e = 0; e < 4; ++e) w[e] = __float_as_uint(v[e]);
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if constexpr (DT == ATTN_F16)
                    w[e] = attn::ptx::pack_f16x2(v[2 * e], v[2 * e + 1]);
                else
                    w[e] = attn::ptx::pack_bf16x2(v[2 * e], v[2 * e + 1]);
            }
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
};

// ---------------------------------------------------------------- reductions
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Max (SUM = false) or sum (SUM = true) over the CTA; `red` holds 32 floats.
template <bool SUM>
__device__ __forceinline__ float block_reduce(float v, float* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nw = static_cast<int>(blockDim.x) >> 5;
    v = SUM ? warp_sum(v) : warp_max(v);
    __syncthreads();  // `red` may still be read from the previous reduction
    if (lane == 0) red[warp] = v;
    __syncthreads();
    v = lane < nw ? red[lane] : (SUM ? 0.f : -INFINITY);
    return SUM ? warp_sum(v) : warp_max(v);
}

// Online (max, sum) pair: sum is relative to max.
__device__ __forceinline__ void online_add(float& m, float& s, float x) {
    if (x > m) {
        s = s * attn::ptx::ex2((m - x) * kLog2e) + 1.f;
        m = x;
    } else {
        s += attn::ptx::ex2((x - m) * kLog2e);
    }
}
__device__ __forceinline__ void online_merge(float& m, float& s, float m2, float s2) {
    const float mx = fmaxf(m, m2);
    if (mx == -INFINITY) return;
    s = s * attn::ptx::ex2((m - mx) * kLog2e) + s2 * attn::ptx::ex2((m2 - mx) * kLog2e);
    m = mx;
}

// ---------------------------------------------------------------- kernels
// A row per warp, CPL 16-byte chunks per lane held in registers.
template <int DT, int CPL>
__global__ void __launch_bounds__(256) softmax_warp_rows(const void* __restrict__ x,
                                                         void* __restrict__ y, int64_t rows,
                                                         int chunks) {
    using C = Chunk<DT>;
    constexpr int EPV = C::EPV;
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < rows;
         r += nwarps) {
        const uint4* src = reinterpret_cast<const uint4*>(x) + r * chunks;
        uint4* dst = reinterpret_cast<uint4*>(y) + r * chunks;
        uint4 c[CPL];
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const int idx = lane + 32 * i;
            c[i] = idx < chunks ? __ldcs(src + idx) : make_uint4(0u, 0u, 0u, 0u);
        }
        float m = -INFINITY;
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            if (lane + 32 * i < chunks) {
                float v[EPV];
                C::unpack(c[i], v);
#pragma unroll
                for (int e = 0; e < EPV; ++e) m = fmaxf(m, v[e]);
            }
        }
        m = warp_max(m);
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            if (lane + 32 * i < chunks) {
                float v[EPV];
                C::unpack(c[i], v);
#pragma unroll
                for (int e = 0; e < EPV; ++e) s += attn::ptx::ex2((v[e] - m) * kLog2e);
            }
        }
        const float inv = 1.f / warp_sum(s);
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const int idx = lane + 32 * i;
            if (idx < chunks) {
                float v[EPV];
                C::unpack(c[i], v);
#pragma unroll
                for (int e = 0; e < EPV; ++e) v[e] = attn::ptx::ex2((v[e] - m) * kLog2e) * inv;
                __stcs(dst + idx, C::pack(v));
            }
        }
    }
}

// A row per CTA of THREADS threads, CPT 16-byte chunks per thread held in registers.
template <int DT, int CPT, int THREADS>
__global__ void __launch_bounds__(THREADS) softmax_cta_rows(const void* __restrict__ x,
                                                            void* __restrict__ y, int64_t rows,
                                                            int chunks) {
    using C = Chunk<DT>;
    constexpr int EPV = C::EPV;
    __shared__ float red[32];
    const int tid = threadIdx.x;
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        const uint4* src = reinterpret_cast<const uint4*>(x) + r * chunks;
        uint4* dst = reinterpret_cast<uint4*>(y) + r * chunks;
        uint4 c[CPT];
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
            const int idx = tid + THREADS * i;
            c[i] = idx < chunks ? __ldcs(src + idx) : make_uint4(0u, 0u, 0u, 0u);
        }
        float m = -INFINITY;
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
            if (tid + THREADS * i < chunks) {
                float v[EPV];
                C::unpack(c[i], v);
#pragma unroll
                for (int e = 0; e < EPV; ++e) m = fmaxf(m, v[e]);
            }
        }
        m = block_reduce<false>(m, red);
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
            if (tid + THREADS * i < chunks) {
                float v[EPV];
                C::unpack(c[i], v);
#pragma unroll
                for (int e = 0; e < EPV; ++e) s += attn::ptx::ex2((v[e] - m) * kLog2e);
            }
        }
        const float inv = 1.f / block_reduce<true>(s, red);
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
            const int idx = tid + THREADS * i;
            if (idx < chunks) {
                float v[EPV];
                C::unpack(c[i], v);
#pragma unroll
                for (int e = 0; e < EPV; ++e) v[e] = attn::ptx::ex2((v[e] - m) * kLog2e) * inv;
                __stcs(dst + idx, C::pack(v));
            }
        }
    }
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}
// Every thread of every CTA of the cluster arrives; shared-memory writes before it
// are visible to the cluster's loads after it.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
                 ::: "memory");
}
// A float in the shared memory of CTA `rank` of the cluster.
__device__ __forceinline__ float ld_cluster_f32(const float* p, uint32_t rank) {
    uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p)), r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(r) : "memory");
    return v;
}

// Rows of any length and alignment: a cluster of CTAs per row (cluster c takes rows
// c, c + #clusters, ...), CTA `rank` the slice [rank * per, (rank + 1) * per) of each
// row, in 16-byte chunks (VEC) or elements.  Two passes over the slice with an
// exchange of (max, sum) pairs between them.
template <int DT, bool VEC>
__global__ void __launch_bounds__(1024) softmax_cluster_rows(const void* __restrict__ x,
                                                             void* __restrict__ y, int64_t rows,
                                                             int n) {
    using E = Elem<DT>;
    using C = Chunk<DT>;
    constexpr int EPV = C::EPV;
    __shared__ float red_m[32], red_s[32];
    __shared__ float part[2];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nw = static_cast<int>(blockDim.x) >> 5;
    const uint32_t rank = cluster_rank(), csize = cluster_size();
    const int64_t n_clusters = gridDim.x / csize;
    const int units = VEC ? n / EPV : n;  // chunks or elements per row
    const int per = (units + static_cast<int>(csize) - 1) / static_cast<int>(csize);
    const int beg = static_cast<int>(rank) * per;
    const int end = min(units, beg + per);
    for (int64_t r = blockIdx.x / csize; r < rows; r += n_clusters) {
        float m = -INFINITY, s = 0.f;
        if constexpr (VEC) {
            // four 16-byte loads in flight per thread before they are used
            const uint4* src = reinterpret_cast<const uint4*>(x) + r * units;
            const int step = static_cast<int>(blockDim.x);
            for (int u0 = beg + tid; u0 < end; u0 += 4 * step) {
                uint4 c[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    c[i] = u0 + i * step < end ? __ldcg(src + u0 + i * step) : make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    if (u0 + i * step < end) {
                        float v[EPV];
                        C::unpack(c[i], v);
#pragma unroll
                        for (int e = 0; e < EPV; ++e) online_add(m, s, v[e]);
                    }
                }
            }
        } else {
            for (int u = beg + tid; u < end; u += blockDim.x) online_add(m, s, E::get(x, r * n + u));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
            const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
            online_merge(m, s, m2, s2);
        }
        if (lane == 0) {
            red_m[warp] = m;
            red_s[warp] = s;
        }
        __syncthreads();
        if (warp == 0) {
            m = lane < nw ? red_m[lane] : -INFINITY;
            s = lane < nw ? red_s[lane] : 0.f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
                const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
                online_merge(m, s, m2, s2);
            }
            if (lane == 0) {
                part[0] = m;
                part[1] = s;
            }
        }
        cluster_sync();  // every CTA's pair is written
        m = -INFINITY;
        s = 0.f;
        for (uint32_t q = 0; q < csize; ++q)
            online_merge(m, s, ld_cluster_f32(&part[0], q), ld_cluster_f32(&part[1], q));
        cluster_sync();  // every CTA has read the pairs: they may be overwritten
        const float inv = 1.f / s;
        if constexpr (VEC) {
            const uint4* src = reinterpret_cast<const uint4*>(x) + r * units;
            uint4* dst = reinterpret_cast<uint4*>(y) + r * units;
            const int step = static_cast<int>(blockDim.x);
            for (int u0 = beg + tid; u0 < end; u0 += 4 * step) {
                uint4 c[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    c[i] = u0 + i * step < end ? __ldcs(src + u0 + i * step) : make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    if (u0 + i * step < end) {
                        float v[EPV];
                        C::unpack(c[i], v);
#pragma unroll
                        for (int e = 0; e < EPV; ++e)
                            v[e] = attn::ptx::ex2((v[e] - m) * kLog2e) * inv;
                        __stcs(dst + u0 + i * step, C::pack(v));
                    }
                }
            }
        } else {
            for (int u = beg + tid; u < end; u += blockDim.x)
                E::put(y, r * n + u, attn::ptx::ex2((E::get(x, r * n + u) - m) * kLog2e) * inv);
        }
    }
}

// ---------------------------------------------------------------- launch
// SM count of the current device, -1 when it is not an sm_100 device.
int num_sms() {
    static int g_num_sms[64];
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return -1;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (g_num_sms[dev] == 0) {
        int major = 0, n = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            return -1;
        }
        g_num_sms[dev] = (major == 10 && n > 0) ? n : -1;
    }
    return g_num_sms[dev];
}

// Persistent grid: resident CTAs per SM x SMs, at most `groups` CTAs.
template <typename K>
int persistent_grid(K kernel, int threads, int64_t groups, int sms) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, 0) != cudaSuccess ||
        per_sm < 1) {
        cudaGetLastError();
        per_sm = 1;
    }
    const int64_t g = static_cast<int64_t>(per_sm) * sms;
    return static_cast<int>(groups < g ? groups : g);
}

template <int DT, int CPL>
int launch_warp(const void* x, void* y, int64_t rows, int chunks, int sms, cudaStream_t s) {
    auto k = softmax_warp_rows<DT, CPL>;
    const int grid = persistent_grid(k, 256, (rows + 7) / 8, sms);
    k<<<grid, 256, 0, s>>>(x, y, rows, chunks);
    return ATTN_OK;
}

template <int DT, int CPT, int THREADS>
int launch_cta(const void* x, void* y, int64_t rows, int chunks, int sms, cudaStream_t s) {
    auto k = softmax_cta_rows<DT, CPT, THREADS>;
    const int grid = persistent_grid(k, THREADS, rows, sms);
    k<<<grid, THREADS, 0, s>>>(x, y, rows, chunks);
    return ATTN_OK;
}

// Cluster size: one CTA per 64 KB of row, up to 8 (the portable limit; clusters of 16
// measured slower here); threads: up to 1024, fewer for short rows.  Grid: as many
// clusters as can be resident at once, at most one per row.  (Capping the rows in
// flight so that the second pass reads from L2 also measured slower: it idles SMs.)
template <int DT, bool VEC>
int launch_cluster(const void* x, void* y, int64_t rows, int n, int sms, cudaStream_t s) {
    const int64_t bytes = static_cast<int64_t>(n) * Elem<DT>::kBytes;
    auto k = softmax_cluster_rows<DT, VEC>;
    constexpr int cmax = 8;
    int csize = 1;
    while (csize < cmax && bytes > static_cast<int64_t>(csize) * 65536) csize *= 2;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    int max_clusters = 0;
    for (;; csize /= 2) {
        const int64_t per_cta = (static_cast<int64_t>(n) + csize - 1) / csize;
        const int threads = per_cta >= 1024 ? 1024 : static_cast<int>((per_cta + 31) / 32 * 32);
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = static_cast<unsigned>(csize);
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg = cudaLaunchConfig_t{};
        cfg.blockDim = dim3(static_cast<unsigned>(threads));
        cfg.gridDim = dim3(static_cast<unsigned>(csize));
        cfg.dynamicSmemBytes = 0;
        cfg.stream = s;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&max_clusters, k, &cfg) != cudaSuccess) {
            cudaGetLastError();
            max_clusters = 0;
        }
        if (max_clusters >= 1 || csize == 1) break;  // a cluster this size fits, or none
    }
    if (max_clusters < 1) max_clusters = sms;
    const int64_t clusters = rows < max_clusters ? rows : max_clusters;
    cfg.gridDim = dim3(static_cast<unsigned>(clusters * csize));
    if (cudaLaunchKernelEx(&cfg, k, x, y, rows, n) != cudaSuccess) {
        cudaGetLastError();
        return ATTN_ERR_LAUNCH;
    }
    return ATTN_OK;
}

template <int DT>
int launch_dt(const void* x, void* y, int64_t rows, int n, int sms, cudaStream_t s) {
    constexpr int esz = Elem<DT>::kBytes;
    const bool vec = (static_cast<int64_t>(n) * esz) % 16 == 0 &&
                     (reinterpret_cast<uintptr_t>(x) & 15u) == 0 &&
                     (reinterpret_cast<uintptr_t>(y) & 15u) == 0;
    if (vec) {
        const int chunks = static_cast<int>(static_cast<int64_t>(n) * esz / 16);
        if (chunks <= 32) return launch_warp<DT, 1>(x, y, rows, chunks, sms, s);
        if (chunks <= 64) return launch_warp<DT, 2>(x, y, rows, chunks, sms, s);
        if (chunks <= 128) return launch_warp<DT, 4>(x, y, rows, chunks, sms, s);
        if (chunks <= 256) return launch_warp<DT, 8>(x, y, rows, chunks, sms, s);
        if (chunks <= 512) return launch_warp<DT, 16>(x, y, rows, chunks, sms, s);
        if (chunks <= 1024) return launch_cta<DT, 4, 256>(x, y, rows, chunks, sms, s);
        if (chunks <= 2048) return launch_cta<DT, 4, 512>(x, y, rows, chunks, sms, s);
        if (chunks <= 4096) return launch_cta<DT, 8, 512>(x, y, rows, chunks, sms, s);
        if (chunks <= 8192) return launch_cta<DT, 8, 1024>(x, y, rows, chunks, sms, s);
    }
    return vec ? launch_cluster<DT, true>(x, y, rows, n, sms, s)
               : launch_cluster<DT, false>(x, y, rows, n, sms, s);
}

}  // namespace

extern "C" {

int row_softmax(const void* x, void* y, long long rows, int n, int dtype, attn_stream_t stream) {
    if (rows < 0 || n < 1 || n > ROW_SOFTMAX_MAX_N) return ATTN_ERR_SHAPE;
    if (dtype != ATTN_F16 && dtype != ATTN_BF16 && dtype != SOFTMAX_F32) return ATTN_ERR_DTYPE;
    if (rows == 0) return ATTN_OK;
    if (!x || !y) return ATTN_ERR_NULLPTR;
    const int esz = dtype == SOFTMAX_F32 ? 4 : 2;
    if ((reinterpret_cast<uintptr_t>(x) % esz) != 0 || (reinterpret_cast<uintptr_t>(y) % esz) != 0)
        return ATTN_ERR_ALIGN;
    const uintptr_t bytes = static_cast<uintptr_t>(rows) * static_cast<uintptr_t>(n) * esz;
    const uintptr_t a = reinterpret_cast<uintptr_t>(x), b = reinterpret_cast<uintptr_t>(y);
    if (a != b && a < b + bytes && b < a + bytes) return ATTN_ERR_ALIAS;
    const int sms = num_sms();
    if (sms < 1) return ATTN_ERR_DEVICE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int64_t r = static_cast<int64_t>(rows);
    int rc;
    if (dtype == ATTN_F16)
        rc = launch_dt<ATTN_F16>(x, y, r, n, sms, s);
    else if (dtype == ATTN_BF16)
        rc = launch_dt<ATTN_BF16>(x, y, r, n, sms, s);
    else
        rc = launch_dt<SOFTMAX_F32>(x, y, r, n, sms, s);
    if (rc != ATTN_OK) return rc;
    return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH;
}

}  // extern "C"
