// lf_select.cu -- two-level mask selection of one HSA call ("Light Forcing：通过
// 稀疏注意力加速自回归视频扩散", paper.rainbus.top, execution flow, stage 3:
// frame scores p_r = <q~_r, k^_M> and top-k frames T_r with the sink, most
// recent and current-chunk frames always kept; block scores
// o_r(tau,j) = <q~_r, k~_j^(tau)> and top-k blocks J_r(tau) in each selected
// frame, giving the mask B_r(tau,j) = 1[tau in T_r, j in J_r(tau)];
// gist.science Technical Summary 2.2 "Two-Level Mask Selection").
//
// Latency-bound (a few MB of pooled fp32 data, read from L2). One warp per
// scored row:
//   * scores: each lane holds head_dim/32 coordinates of q~_r; for a group of
//     32 candidates each lane forms its 32 partial products and a butterfly
//     "transpose reduce" (31 shuffles) leaves candidate c's full inner product
//     in lane c;
//   * ranking: a candidate is the 64-bit key (orderable(score) << 32) |
//     (0xFFFFFFFF - index), so a larger key is a larger score, and among equal
//     scores the lower index; keys are unique.
//   * frames: top-k by k rounds of warp arg-max over the keys;
//   * blocks: top-k by rank counting (rank = number of larger keys), then a
//     ballot/popc compaction writes the kept block ids in ascending order.
// The one-dimensional variant (global block top-k, no frame level) takes one
// CTA per scored row instead; see select_blocks_1d_kernel.
#include "lf_device.cuh"
#include "lf_internal.h"
#include "lf_score.cuh"

namespace lf {
namespace {

constexpr int SEL_THREADS = 256;
constexpr int SEL_WARPS = SEL_THREADS / 32;

// KPL = key slots per lane = ceil(n_mem / 32).
template <int D, int KPL>
__global__ void __launch_bounds__(SEL_THREADS) select_frames_kernel(const SelectFramesArgs a)
{
    constexpr int EPL = D / 32;
    const int lane = threadIdx.x & 31;
    const long long row = static_cast<long long>(blockIdx.x) * SEL_WARPS + (threadIdx.x >> 5);
    if (row >= static_cast<long long>(a.BH) * a.Rq) return;
    int* out = a.frame_sel + row * a.n_sel;
    if (a.chunk_index == 1) {
        for (int t = lane; t < a.NF; t += 32) out[t] = t;
        return;
    }
    const int bh = static_cast<int>(row / a.Rq);
    const int n_mem = a.NF - a.n_sink - a.n_recent - a.n_cur;
    const int kf = a.topk < n_mem ? a.topk : n_mem;

    float qv[EPL];
    load_lane<EPL>(qv, a.q_pool + row * D + lane * EPL);
    const float* kmem = a.k_frame + (static_cast<long long>(bh) * a.NF + a.n_sink) * D;

    uint64_t key[KPL];
#pragma unroll
    for (int i = 0; i < KPL; ++i) {
        const float sc = score_group<D>(qv, kmem, i * 32, n_mem, lane);
        const int m = i * 32 + lane;
        key[i] = (m < n_mem) ? make_key(sc, m) : 0ull;
    }

    uint32_t sel = 0;  // bit i: key slot i of this lane is in the top-k
    for (int t = 0; t < kf; ++t) {
        uint64_t best = 0;
#pragma unroll
        for (int i = 0; i < KPL; ++i) best = key[i] > best ? key[i] : best;
        const uint64_t wbest = warp_max_u64(best);
#pragma unroll
        for (int i = 0; i < KPL; ++i)
            if (key[i] == wbest && wbest != 0ull) {
                sel |= 1u << i;
                key[i] = 0ull;
            }
    }

    // T_r = sinks, selected memory frames (ascending), recent + current frames.
    for (int t = lane; t < a.n_sink; t += 32) out[t] = t;
    int prefix = a.n_sink;
    const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
    for (int i = 0; i < KPL; ++i) {
        const bool s = (sel >> i) & 1u;
        const uint32_t mask = __ballot_sync(0xffffffffu, s);
        if (s) out[prefix + __popc(mask & lt)] = a.n_sink + i * 32 + lane;
        prefix += __popc(mask);
    }
    const int tail0 = a.NF - a.n_recent - a.n_cur;
    for (int t = lane; t < a.n_recent + a.n_cur; t += 32) out[a.n_sink + kf + t] = tail0 + t;
}

// One warp per (row, selected-frame slot). KPL = ceil(bpf / 32).
template <int D, int KPL>
__global__ void __launch_bounds__(SEL_THREADS) select_blocks_kernel(const SelectBlocksArgs a)
{
    constexpr int EPL = D / 32;
    const int lane = threadIdx.x & 31;
    const long long gw = static_cast<long long>(blockIdx.x) * SEL_WARPS + (threadIdx.x >> 5);
    if (gw >= static_cast<long long>(a.BH) * a.Rq * a.n_sel) return;
    const long long row = gw / a.n_sel;
    const int s = static_cast<int>(gw - row * a.n_sel);
    const int bh = static_cast<int>(row / a.Rq);
    int* out = a.block_list + row * a.list_cap + static_cast<long long>(s) * a.kb;
    if (s == 0 && lane == 0) a.block_count[row] = a.n_sel * a.kb;

    const int tau = (a.chunk_index == 1) ? s : __ldg(a.frame_sel + row * a.n_sel + s);
    if (tau < 0 || tau >= a.NF) {
        // A frame id outside the call: write ids the attention kernel rejects.
        for (int t = lane; t < a.kb; t += 32) out[t] = -1;
        if (lane == 0) record_error(a.err, DEVERR_LIST | 3);
        return;
    }

    float qv[EPL];
    load_lane<EPL>(qv, a.q_pool + row * D + lane * EPL);
    const float* kblk = a.k_pool + (static_cast<long long>(bh) * a.NF * a.bpf + static_cast<long long>(tau) * a.bpf) * D;

    uint64_t key[KPL];
#pragma unroll
    for (int i = 0; i < KPL; ++i) {
        const float sc = score_group<D>(qv, kblk, i * 32, a.bpf, lane);
        const int j = i * 32 + lane;
        key[i] = (j < a.bpf) ? make_key(sc, j) : 0ull;
    }

    int rank[KPL];
#pragma unroll
    for (int i = 0; i < KPL; ++i) rank[i] = 0;
    for (int src = 0; src < 32; ++src) {
#pragma unroll
        for (int i2 = 0; i2 < KPL; ++i2) {
            const uint64_t o = __shfl_sync(0xffffffffu, key[i2], src);
#pragma unroll
            for (int i = 0; i < KPL; ++i) rank[i] += (o > key[i]) ? 1 : 0;
        }
    }

    int prefix = 0;
    const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
    for (int i = 0; i < KPL; ++i) {
        const bool keep = key[i] != 0ull && rank[i] < a.kb;
        const uint32_t mask = __ballot_sync(0xffffffffu, keep);
        if (keep) out[prefix + __popc(mask & lt)] = tau * a.bpf + i * 32 + lane;
        prefix += __popc(mask);
    }
}

// One-dimensional selection (the single-granularity variant of the ablation in
// "南洋理工大学打造视频生成新引擎", 163.com, section 4): one CTA per scored row,
// every KV block of the head a candidate. Warps score groups of 32 candidates
// into 64-bit keys in shared memory; the kb-th largest key T is built bit by
// bit from the top (a candidate bit stays when at least kb keys are >= the
// value with it set; keys are unique, so exactly kb keys are >= T); a ballot
// compaction in index order writes the kept ids ascending.
template <int D>
__global__ void __launch_bounds__(SEL_THREADS) select_blocks_1d_kernel(const SelectBlocks1dArgs a)
{
    constexpr int EPL = D / 32;
    extern __shared__ uint64_t keys[];  // [Nkv]
    __shared__ int red[2][SEL_WARPS];   // per-warp partial counts, two alternating slots
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long row = blockIdx.x;
    const int bh = static_cast<int>(row / a.Rq);
    const int n = a.Nkv;
    int* out = a.block_list + row * a.list_cap;
    const int keep = (a.chunk_index == 1 || a.kb >= n) ? n : a.kb;
    if (tid == 0) a.block_count[row] = keep;
    if (keep == n) {
        for (int g = tid; g < n; g += SEL_THREADS) out[g] = g;
        return;
    }
    float qv[EPL];
    load_lane<EPL>(qv, a.q_pool + row * D + lane * EPL);
    const float* kblk = a.k_pool + static_cast<long long>(bh) * n * D;
    for (int grp = warp; grp * 32 < n; grp += SEL_WARPS) {
        const float sc = score_group<D>(qv, kblk, grp * 32, n, lane);
        const int g = grp * 32 + lane;
        if (g < n) keys[g] = make_key(sc, g);
    }
    __syncthreads();
    uint64_t T = 0;
    for (int bit = 63; bit >= 0; --bit) {
        const uint64_t cand = T | (1ull << bit);
        unsigned c = 0;
        for (int g = tid; g < n; g += SEL_THREADS) c += keys[g] >= cand ? 1u : 0u;
        c = __reduce_add_sync(0xffffffffu, c);
        const int buf = bit & 1;
        if (lane == 0) red[buf][warp] = static_cast<int>(c);
        __syncthreads();
        int total = 0;
#pragma unroll
        for (int w = 0; w < SEL_WARPS; ++w) total += red[buf][w];
        if (total >= keep) T = cand;
    }
    __syncthreads();  // the last round's counts are read before the slots are reused
    int prefix = 0;
    const uint32_t lt = (1u << lane) - 1u;
    for (int base = 0, it = 0; base < n; base += SEL_THREADS, ++it) {
        const int g = base + tid;
        const bool sel = g < n && keys[g] >= T;
        const uint32_t m = __ballot_sync(0xffffffffu, sel);
        const int buf = it & 1;
        if (lane == 0) red[buf][warp] = __popc(m);
        __syncthreads();
        int before = 0, total = 0;
#pragma unroll
        for (int w = 0; w < SEL_WARPS; ++w) {
            const int v = red[buf][w];
            total += v;
            before += (w < warp) ? v : 0;
        }
        if (sel) out[prefix + before + __popc(m & lt)] = g;
        prefix += total;
    }
}

template <int D>
cudaError_t launch_blocks_1d_d(const SelectBlocks1dArgs& a, cudaStream_t s)
{
    const size_t smem = static_cast<size_t>(a.Nkv) * sizeof(uint64_t);
    static int configured_device = -1;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (configured_device != dev) {
        e = cudaFuncSetAttribute(select_blocks_1d_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(SEL1D_MAX_NKV * sizeof(uint64_t)));
        if (e != cudaSuccess) return e;
        configured_device = dev;
    }
    const unsigned grid = static_cast<unsigned>(static_cast<long long>(a.BH) * a.Rq);
    select_blocks_1d_kernel<D><<<grid, SEL_THREADS, smem, s>>>(a);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_frames_d(const SelectFramesArgs& a, unsigned grid, cudaStream_t s)
{
    const int n_mem = a.NF - a.n_sink - a.n_recent - a.n_cur;
    const int kpl = (n_mem + 31) / 32;
    if (a.chunk_index == 1 || kpl <= 1) select_frames_kernel<D, 1><<<grid, SEL_THREADS, 0, s>>>(a);
    else if (kpl <= 2) select_frames_kernel<D, 2><<<grid, SEL_THREADS, 0, s>>>(a);
    else if (kpl <= 4) select_frames_kernel<D, 4><<<grid, SEL_THREADS, 0, s>>>(a);
    else if (kpl <= 8) select_frames_kernel<D, 8><<<grid, SEL_THREADS, 0, s>>>(a);
    else if (kpl <= 16) select_frames_kernel<D, 16><<<grid, SEL_THREADS, 0, s>>>(a);
    else select_frames_kernel<D, 32><<<grid, SEL_THREADS, 0, s>>>(a);
    return cudaGetLastError();
}

template <int D>
cudaError_t launch_blocks_d(const SelectBlocksArgs& a, unsigned grid, cudaStream_t s)
{
    const int kpl = (a.bpf + 31) / 32;
    if (kpl <= 1) select_blocks_kernel<D, 1><<<grid, SEL_THREADS, 0, s>>>(a);
    else if (kpl <= 2) select_blocks_kernel<D, 2><<<grid, SEL_THREADS, 0, s>>>(a);
    else select_blocks_kernel<D, 4><<<grid, SEL_THREADS, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select_blocks_1d(const SelectBlocks1dArgs& a, cudaStream_t s)
{
    if (static_cast<long long>(a.BH) * a.Rq <= 0) return cudaSuccess;
    return a.D == 128 ? launch_blocks_1d_d<128>(a, s) : launch_blocks_1d_d<64>(a, s);
}

cudaError_t launch_select_frames(const SelectFramesArgs& a, cudaStream_t s)
{
    const long long rows = static_cast<long long>(a.BH) * a.Rq;
    if (rows <= 0) return cudaSuccess;
    const unsigned grid = static_cast<unsigned>((rows + SEL_WARPS - 1) / SEL_WARPS);
    return a.D == 128 ? launch_frames_d<128>(a, grid, s) : launch_frames_d<64>(a, grid, s);
}

cudaError_t launch_select_blocks(const SelectBlocksArgs& a, cudaStream_t s)
{
    const long long warps = static_cast<long long>(a.BH) * a.Rq * a.n_sel;
    if (warps <= 0) return cudaSuccess;
    const unsigned grid = static_cast<unsigned>((warps + SEL_WARPS - 1) / SEL_WARPS);
    return a.D == 128 ? launch_blocks_d<128>(a, grid, s) : launch_blocks_d<64>(a, grid, s);
}

}  // namespace lf
