// lf_pool.cu -- token compression of one HSA call ("Light Forcing：通过稀疏注意力
// 加速自回归视频扩散", paper.rainbus.top, execution flow, stage 2: block mean
// pooling of q and k, frame-level compression of the keys; gist.science
// Technical Summary 2.2 "Token Compression").
//
// HBM-bound. One CTA per (batch*head, frame): K frames first, then the query
// frames of the current chunk. A frame is streamed block by block (64 tokens x
// head_dim bf16, contiguous) with 128-bit coalesced loads, UNROLL blocks in
// flight per thread. Each block's column sums are reduced with warp shuffles
// inside a warp and then across the CTA's 8 warps in a fixed order through
// shared memory (deterministic). The frame mean is the sum of the frame's block
// sums divided by the frame's token count, so K is read once.
#include "lf_internal.h"

#include <cuda_bf16.h>

namespace lf {
namespace {

constexpr int POOL_THREADS = 256;
constexpr int POOL_WARPS = POOL_THREADS / 32;
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

template <int D, int UNROLL>
__global__ void __launch_bounds__(POOL_THREADS) pool_kernel(const PoolArgs a)
{
    constexpr int CPR = D / 8;                              // 16-byte chunks per token row
    constexpr int RPI = 32 / CPR;                           // rows one warp load covers
    constexpr int ROWS_PER_WARP = BLOCK_TOKENS / POOL_WARPS;  // 8 rows of a block per warp
    constexpr int LOADS = ROWS_PER_WARP / RPI;              // loads per lane per block
    static_assert(LOADS >= 1 && ROWS_PER_WARP % RPI == 0, "layout");
    static_assert(UNROLL * D <= POOL_THREADS, "final reduction needs UNROLL*D threads");

    __shared__ float red[UNROLL][POOL_WARPS][D];
    __shared__ float bsum[UNROLL][D];

    const int units = a.NF + a.n_cur;
    const int bh = blockIdx.x / units;
    const int f = blockIdx.x - bh * units;
    const bool is_k = f < a.NF;
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
    float frame_acc = 0.f;

    for (int j0 = 0; j0 < a.bpf; j0 += UNROLL) {
        uint4 buf[UNROLL][LOADS];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int j = j0 + u;
            const int nrows = (j < a.bpf) ? min(BLOCK_TOKENS, a.F - j * BLOCK_TOKENS) : 0;
#pragma unroll
            for (int l = 0; l < LOADS; ++l) {
                const int row = warp * ROWS_PER_WARP + l * RPI + rsub;
                if (row < nrows)
                    buf[u][l] = ld_stream_v4(src + static_cast<long long>(j * BLOCK_TOKENS + row) * D + chunk * 8);
                else
                    buf[u][l] = make_uint4(0u, 0u, 0u, 0u);
            }
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int l = 0; l < LOADS; ++l) add_bf16x8(acc, buf[u][l]);
#pragma unroll
            for (int off = CPR; off < 32; off <<= 1)
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], off);
            if (rsub == 0) {
#pragma unroll
                for (int i = 0; i < 8; ++i) red[u][warp][chunk * 8 + i] = acc[i];
            }
        }
        __syncthreads();
        if (threadIdx.x < UNROLL * D) {
            const int u = threadIdx.x / D, col = threadIdx.x - u * D;
            const int j = j0 + u;
            float s = 0.f;
#pragma unroll
            for (int w = 0; w < POOL_WARPS; ++w) s += red[u][w][col];
            if (j < a.bpf) {
                const int nrows = min(BLOCK_TOKENS, a.F - j * BLOCK_TOKENS);
                dst[static_cast<long long>(j) * D + col] = s / static_cast<float>(nrows);
            }
            bsum[u][col] = (j < a.bpf) ? s : 0.f;
        }
        __syncthreads();
        if (is_k && threadIdx.x < D) {
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) frame_acc += bsum[u][threadIdx.x];
        }
    }
    if (is_k && threadIdx.x < D)
        a.k_frame[(static_cast<long long>(bh) * a.NF + f) * D + threadIdx.x] = frame_acc / static_cast<float>(a.F);
}

}  // namespace

cudaError_t launch_pool(const PoolArgs& a, cudaStream_t s)
{
    const long long grid = static_cast<long long>(a.BH) * (a.NF + a.n_cur);
    if (grid <= 0) return cudaSuccess;
    if (a.D == 128)
        pool_kernel<128, 2><<<static_cast<unsigned>(grid), POOL_THREADS, 0, s>>>(a);
    else
        pool_kernel<64, 4><<<static_cast<unsigned>(grid), POOL_THREADS, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace lf
