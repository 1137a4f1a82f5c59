// lf_quant.cu -- per-token e4m3 quantisation for the FP8 attention path.
//
// The pages quantise the model's linear layers to FP8 with per-token activation
// scales ("南洋理工大学打造视频生成新引擎", 163.com, deployment section; "Light
// Forcing: Accelerating Autoregressive Video Diffusion via Sparse Attention",
// gist.science, Technical Summary 4, deployment acceleration) and describe no FP8
// attention. Reading taken for the FP8 attention here: Q and K in e4m3 with one
// scale per token (a row of head_dim values), V and the softmax weights in bf16.
//
// Per row: s = fl32(amax / 448) (1 for an all-zero row), code = e4m3(fl32(x / s))
// (round to nearest even, saturating at 448; IEEE fp32 division). The code is a
// decision taken in floating point, so this kernel and the oracle take it in the
// same precision (fp32) and agree bit for bit. HBM-bound: one warp per four rows, each
// lane reads D/32 bf16 values (8 bytes at D = 128) of each of four rows before it
// processes any (more bytes in flight per warp), and writes D/32 codes per row.
#include "lf_internal.h"

#include <cuda_bf16.h>

namespace lf {
namespace {

constexpr int QUANT_THREADS = 256;

__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

constexpr int QUANT_ROWS_PER_WARP = 4;  // rows loaded before any is processed (bytes in flight)

template <int EPL>
__device__ __forceinline__ void load_row_bf16(float (&v)[EPL], const uint16_t* src)
{
    if constexpr (EPL == 4) {
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(src));
        v[0] = __uint_as_float(u.x << 16);
        v[1] = __uint_as_float(u.x & 0xFFFF0000u);
        v[2] = __uint_as_float(u.y << 16);
        v[3] = __uint_as_float(u.y & 0xFFFF0000u);
    } else {
        const uint32_t u = __ldg(reinterpret_cast<const uint32_t*>(src));
        v[0] = __uint_as_float(u << 16);
        v[1] = __uint_as_float(u & 0xFFFF0000u);
    }
}

template <int D>
__global__ void __launch_bounds__(QUANT_THREADS) quant_rows_kernel(const uint16_t* __restrict__ x, long long n_rows,
                                                                   uint8_t* __restrict__ x8, float* __restrict__ scale)
{
    constexpr int EPL = D / 32;  // 4 (head_dim 128) or 2 (head_dim 64)
    constexpr int R = QUANT_ROWS_PER_WARP;
    const int lane = threadIdx.x & 31;
    const long long row0 = (static_cast<long long>(blockIdx.x) * (QUANT_THREADS / 32) + (threadIdx.x >> 5)) * R;
    float v[R][EPL];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        if (row0 + r < n_rows) load_row_bf16<EPL>(v[r], x + (row0 + r) * D + lane * EPL);
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const long long row = row0 + r;
        if (row >= n_rows) break;  // warp-uniform
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < EPL; ++i) amax = fmaxf(amax, fabsf(v[r][i]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float s = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
        uint8_t* dst = x8 + row * D + lane * EPL;
        if constexpr (EPL == 4) {
            const uint32_t c = e4m3x2(__fdiv_rn(v[r][0], s), __fdiv_rn(v[r][1], s)) |
                               (e4m3x2(__fdiv_rn(v[r][2], s), __fdiv_rn(v[r][3], s)) << 16);
            *reinterpret_cast<uint32_t*>(dst) = c;
        } else {
            *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(e4m3x2(__fdiv_rn(v[r][0], s), __fdiv_rn(v[r][1], s)));
        }
        if (lane == 0) scale[row] = s;
    }
}

}  // namespace

cudaError_t launch_quant_rows(const uint16_t* x, long long n_rows, int D, uint8_t* x8, float* scale, cudaStream_t s)
{
    if (n_rows <= 0) return cudaSuccess;
    const long long rows_per_cta = static_cast<long long>(QUANT_THREADS / 32) * QUANT_ROWS_PER_WARP;
    const long long grid = (n_rows + rows_per_cta - 1) / rows_per_cta;
    if (D == 128)
        quant_rows_kernel<128><<<static_cast<unsigned>(grid), QUANT_THREADS, 0, s>>>(x, n_rows, x8, scale);
    else
        quant_rows_kernel<64><<<static_cast<unsigned>(grid), QUANT_THREADS, 0, s>>>(x, n_rows, x8, scale);
    return cudaGetLastError();
}

}  // namespace lf
