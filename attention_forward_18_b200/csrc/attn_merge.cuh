// attn_merge.cuh -- merge of split-KV partial results into the attention output.
//
// A split pass computes, for each KV range s of a (query row, head), the softmax
// attention restricted to that range: O_s (already divided by its own normaliser)
// and LSE_s = ln sum_{j in range s} exp(scale * q.k_j).  The whole-range result is
// the LSE-weighted average
//     LSE = ln sum_s exp(LSE_s),   O = sum_s exp(LSE_s - LSE) O_s,
// which is exact (the weights are each range's share of the full normaliser).
// Ranges with no visible key carry LSE_s = -inf and weight 0.
//
// Memory-bound: one warp per output row; lane l reads D/32 consecutive fp32 values
// of every partial row (a warp reads whole, contiguous rows), the result is rounded
// once to 16 bits.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace attn {

template <int D, bool IS_BF16>
__global__ void __launch_bounds__(256)
    attn_splitkv_merge_kernel(const float* __restrict__ ws_o, const float* __restrict__ ws_lse,
                              void* __restrict__ o, float* __restrict__ lse, int n_splits,
                              int64_t rows) {
    constexpr int V = D / 32;  // values per lane
    const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;

    float mx = -INFINITY;
    for (int s = lane; s < n_splits; s += 32) mx = fmaxf(mx, ws_lse[s * rows + row]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));

    float acc[V];
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = 0.f;
    float wsum = 0.f;
    for (int s = 0; s < n_splits; ++s) {
        const float ls = ws_lse[s * rows + row];
        const float wgt = (ls == -INFINITY) ? 0.f : expf(ls - mx);
        wsum += wgt;
        const float* src = ws_o + (s * rows + row) * D + lane * V;
        if constexpr (V % 4 == 0) {
#pragma unroll
            for (int e = 0; e < V; e += 4) {
                const float4 x = *reinterpret_cast<const float4*>(src + e);
                acc[e] += wgt * x.x;
                acc[e + 1] += wgt * x.y;
                acc[e + 2] += wgt * x.z;
                acc[e + 3] += wgt * x.w;
            }
        } else {
#pragma unroll
            for (int e = 0; e < V; e += 2) {
                const float2 x = *reinterpret_cast<const float2*>(src + e);
                acc[e] += wgt * x.x;
                acc[e + 1] += wgt * x.y;
            }
        }
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    uint32_t packed[V / 2];
#pragma unroll
    for (int e = 0; e < V / 2; ++e) {
        if constexpr (IS_BF16)
            packed[e] = ptx::pack_bf16x2(acc[2 * e] * inv, acc[2 * e + 1] * inv);
        else
            packed[e] = ptx::pack_f16x2(acc[2 * e] * inv, acc[2 * e + 1] * inv);
    }
    uint16_t* dst = reinterpret_cast<uint16_t*>(o) + row * D + lane * V;
    if constexpr (V % 4 == 0) {
#pragma unroll
        for (int e = 0; e < V / 2; e += 2)
            *reinterpret_cast<uint2*>(dst + 2 * e) = make_uint2(packed[e], packed[e + 1]);
    } else {
#pragma unroll
        for (int e = 0; e < V / 2; ++e) *reinterpret_cast<uint32_t*>(dst + 2 * e) = packed[e];
    }
    if (lane == 0 && lse != nullptr) lse[row] = wsum > 0.f ? mx + logf(wsum) : -INFINITY;
}

// The same merge for any head dimension d <= 128 (rows of d values): lane l takes
// columns l, l + 32, l + 64, l + 96 (coalesced across the warp).
template <bool IS_BF16>
__global__ void __launch_bounds__(256)
    attn_splitkv_merge_any_d(const float* __restrict__ ws_o, const float* __restrict__ ws_lse,
                             void* __restrict__ o, float* __restrict__ lse, int n_splits,
                             int64_t rows, int d) {
    const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    float mx = -INFINITY;
    for (int s = lane; s < n_splits; s += 32) mx = fmaxf(mx, ws_lse[s * rows + row]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    float wsum = 0.f;
    for (int s = 0; s < n_splits; ++s) {
        const float ls = ws_lse[s * rows + row];
        const float wgt = (ls == -INFINITY) ? 0.f : expf(ls - mx);
        wsum += wgt;
        const float* src = ws_o + (s * rows + row) * d;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (lane + 32 * i < d) acc[i] += wgt * src[lane + 32 * i];
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    uint16_t* dst = reinterpret_cast<uint16_t*>(o) + row * d;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (lane + 32 * i < d) {
            const uint32_t pk = IS_BF16 ? ptx::pack_bf16x2(acc[i] * inv, 0.f)
                                        : ptx::pack_f16x2(acc[i] * inv, 0.f);
            dst[lane + 32 * i] = static_cast<uint16_t>(pk & 0xffffu);
        }
    }
    if (lane == 0 && lse != nullptr) lse[row] = wsum > 0.f ? mx + logf(wsum) : -INFINITY;
}

}  // namespace attn
