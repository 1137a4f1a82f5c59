// lf_pool.cu -- token compression of one HSA call ("Light Forcing：通过稀疏注意力
// 加速自回归视频扩散", paper.rainbus.top, execution flow, stage 2: block mean
// pooling of q and k, frame-level compression of the keys; gist.science
// Technical Summary 2.2 "Token Compression").
//
// HBM-bound. One CTA per (batch*head, frame): the pooled K frames first, then
// the query frames of the current chunk. The CTA has W warps, W chosen so that it
// divides the frame's block count where possible (5 for the 25 blocks of a 1560-token
// frame), so every warp streams the same number of blocks and none idles at the end.
// Warp w owns blocks w, w+W, w+2W, ... and streams each block (64 tokens x head_dim
// bf16, 16 KB, contiguous) with 128-bit coalesced loads, 16 per lane in flight; a
// block's column sums are reduced with warp shuffles only, so no CTA-wide barrier
// sits between loads. Several small CTAs share an SM, which keeps about 100 KB per SM
// in flight. The frame sum is each warp's running sum of its block sums, combined
// across the warps in a fixed order through shared memory once at the end
// (deterministic), then divided by the frame's token count, so K is read once.
#include "lf_internal.h"

#include <cuda_bf16.h>

namespace lf {
namespace {

constexpr int POOL_MAX_WARPS = 8;
constexpr int BLOCK_TOKENS = 64;

__device__ __forceinline__ uint4 ld_stream_v4(const uint16_t* p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void add_bf16x8(float (&acc)[8], const uint4& u)
{
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] += __uint_as_float(w[i] << 16);
        acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

template <int D>
__global__ void __launch_bounds__(POOL_MAX_WARPS * 32) pool_kernel(const PoolArgs a)
{
    constexpr int CPR = D / 8;          // 16-byte chunks per token row
    constexpr int RPL = 32 / CPR;       // rows one warp-wide load covers
    constexpr int LOADS = BLOCK_TOKENS / RPL;  // loads per lane per block
    constexpr int PHASE = 16;           // loads in flight per lane
    static_assert(LOADS % PHASE == 0, "layout");

    __shared__ float red[POOL_MAX_WARPS][D];
    const int n_warps = blockDim.x >> 5;

    const int units = a.nk + (a.pool_q ? a.n_cur : 0);
    const int bh = blockIdx.x / units;
    const int u = blockIdx.x - bh * units;
    const bool is_k = u < a.nk;
    const int f = is_k ? a.f0 + u : a.NF + (u - a.nk);
    const uint16_t* src;
    float* dst;
    if (is_k) {
        src = a.k + (static_cast<long long>(bh) * a.kv_stride + static_cast<long long>(f) * a.F) * D;
        dst = a.k_pool + (static_cast<long long>(bh) * a.NF * a.bpf + static_cast<long long>(f) * a.bpf) * D;
    } else {
        const int fq = f - a.NF;
        src = a.q + (static_cast<long long>(bh) * a.n_cur * a.F + static_cast<long long>(fq) * a.F) * D;
        dst = a.q_pool + (static_cast<long long>(bh) * a.n_cur * a.bpf + static_cast<long long>(fq) * a.bpf) * D;
    }

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int chunk = lane % CPR, rsub = lane / CPR;
    float facc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // this warp's share of the frame sum

    for (int j = warp; j < a.bpf; j += n_warps) {
        const int nrows = min(BLOCK_TOKENS, a.F - j * BLOCK_TOKENS);
        const uint16_t* bsrc = src + static_cast<long long>(j) * BLOCK_TOKENS * D + chunk * 8;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int ph = 0; ph < LOADS / PHASE; ++ph) {
            uint4 buf[PHASE];
#pragma unroll
            for (int i = 0; i < PHASE; ++i) {
                const int row = (ph * PHASE + i) * RPL + rsub;
                buf[i] = row < nrows ? ld_stream_v4(bsrc + static_cast<long long>(row) * D) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int i = 0; i < PHASE; ++i) add_bf16x8(acc, buf[i]);
        }
#pragma unroll
        for (int off = CPR; off < 32; off <<= 1)
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], off);
        if (rsub == 0) {
            float4* o = reinterpret_cast<float4*>(dst + static_cast<long long>(j) * D + chunk * 8);
            const float n = static_cast<float>(nrows);
            o[0] = make_float4(acc[0] / n, acc[1] / n, acc[2] / n, acc[3] / n);
            o[1] = make_float4(acc[4] / n, acc[5] / n, acc[6] / n, acc[7] / n);
#pragma unroll
            for (int i = 0; i < 8; ++i) facc[i] += acc[i];
        }
    }
    if (!is_k) return;
    if (rsub == 0) {
#pragma unroll
        for (int i = 0; i < 8; ++i) red[warp][chunk * 8 + i] = facc[i];
    }
    __syncthreads();
    for (int c = threadIdx.x; c < D; c += blockDim.x) {
        float s = 0.f;
        for (int w = 0; w < n_warps; ++w) s += red[w][c];
        a.k_frame[(static_cast<long long>(bh) * a.NF + f) * D + c] = s / static_cast<float>(a.F);
    }
}

}  // namespace

// Warps per CTA: the count in 4..8 that leaves the fewest idle warp-blocks over the
// frame's bpf blocks (ties to more warps); frames of fewer than 4 blocks get one warp
// per block. bpf = 25 gives 5 (no idle warp), bpf = 24 gives 8, bpf = 4 gives 4.
int pool_warps(int bpf)
{
    if (bpf < 4) return bpf < 1 ? 1 : bpf;
    int best = POOL_MAX_WARPS, waste = 1 << 30;
    for (int w = POOL_MAX_WARPS; w >= 4; --w) {
        const int idle = ((bpf + w - 1) / w) * w - bpf;
        if (idle < waste) {
            waste = idle;
            best = w;
        }
    }
    return best;
}

cudaError_t launch_pool(const PoolArgs& a, cudaStream_t s)
{
    const long long grid = static_cast<long long>(a.BH) * (a.nk + (a.pool_q ? a.n_cur : 0));
    if (grid <= 0) return cudaSuccess;
    const int threads = 32 * pool_warps(a.bpf);
    if (a.D == 128)
        pool_kernel<128><<<static_cast<unsigned>(grid), threads, 0, s>>>(a);
    else
        pool_kernel<64><<<static_cast<unsigned>(grid), threads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace lf
