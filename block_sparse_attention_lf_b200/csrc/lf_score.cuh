// lf_score.cuh -- warp-level scoring helpers shared by the selection kernels
// (lf_select.cu, lf_ivf.cu): fp32 inner products of a query block mean with 32
// candidate rows at a time, and the 64-bit ranking keys. Every selection kernel
// forms a candidate's score with the same partial products and the same reduction
// tree, so a given (query block, candidate) pair scores the same bits in each.
#pragma once

#include "lf_device.cuh"

namespace lf {

// After the call lane c holds sum over lanes of v[c] in v[0].
__device__ __forceinline__ void transpose_reduce_sum(float (&v)[32], int lane)
{
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) {
        const bool upper = (lane & s) != 0;
#pragma unroll
        for (int i = 0; i < s; ++i) {
            const float send = upper ? v[i] : v[i + s];
            const float keep = upper ? v[i + s] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
        }
    }
}

// SHARED: p points into shared memory (plain load); otherwise read-only global memory.
template <int EPL, bool SHARED = false>
__device__ __forceinline__ void load_lane(float (&dst)[EPL], const float* p)
{
    if constexpr (EPL == 4) {
        const float4 t = SHARED ? *reinterpret_cast<const float4*>(p) : __ldg(reinterpret_cast<const float4*>(p));
        dst[0] = t.x; dst[1] = t.y; dst[2] = t.z; dst[3] = t.w;
    } else {
        const float2 t = SHARED ? *reinterpret_cast<const float2*>(p) : __ldg(reinterpret_cast<const float2*>(p));
        dst[0] = t.x; dst[1] = t.y;
    }
}

// Scores of candidates base..base+31 (rows of `rows`, D floats each, only the
// first n are real; in shared memory when SHARED); returns the score of candidate
// base+lane (0 if beyond n).
template <int D, bool SHARED = false>
__device__ __forceinline__ float score_group(const float (&qv)[D / 32], const float* rows, int base,
                                             int n, int lane)
{
    constexpr int EPL = D / 32;
    float part[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) {
        part[c] = 0.f;
        if (base + c < n) {
            float kv[EPL];
            load_lane<EPL, SHARED>(kv, rows + static_cast<long long>(base + c) * D + lane * EPL);
#pragma unroll
            for (int e = 0; e < EPL; ++e) part[c] = fmaf(qv[e], kv[e], part[c]);
        }
    }
    transpose_reduce_sum(part, lane);
    return part[0];
}

__device__ __forceinline__ uint64_t make_key(float score, int idx)
{
    return (static_cast<uint64_t>(orderable(score)) << 32) | static_cast<uint64_t>(0xFFFFFFFFu - static_cast<uint32_t>(idx));
}

__device__ __forceinline__ uint64_t warp_max_u64(uint64_t v)
{
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        const uint64_t o = __shfl_xor_sync(0xffffffffu, v, off);
        v = o > v ? o : v;
    }
    return v;
}

}  // namespace lf
