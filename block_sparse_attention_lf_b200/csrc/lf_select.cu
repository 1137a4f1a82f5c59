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
constexpr int SEL_FUSED_MAX_WARPS = 16;

// T_r of scored row `row` (one warp): frame scores of the memory frames, top-k_f by
// warp arg-max rounds, forced frames added; written ascending to out (global) and, when
// sel_copy is not NULL, to sel_copy too. KPL = key slots per lane = ceil(n_mem / 32).
template <int D, int KPL>
__device__ __forceinline__ void frames_of_row(const SelectFramesArgs& a, long long row, int lane, const float (&qv)[D / 32],
                                              int* out, int* sel_copy)
{
    if (a.chunk_index == 1) {
        for (int t = lane; t < a.NF; t += 32) {
            out[t] = t;
            if (sel_copy) sel_copy[t] = t;
        }
        return;
    }
    const int bh = static_cast<int>(row / a.Rq);
    const int n_mem = a.NF - a.n_sink - a.n_recent - a.n_cur;
    const int kf = a.topk < n_mem ? a.topk : n_mem;
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
    for (int t = lane; t < a.n_sink; t += 32) {
        out[t] = t;
        if (sel_copy) sel_copy[t] = t;
    }
    int prefix = a.n_sink;
    const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
    for (int i = 0; i < KPL; ++i) {
        const bool s = (sel >> i) & 1u;
        const uint32_t mask = __ballot_sync(0xffffffffu, s);
        if (s) {
            out[prefix + __popc(mask & lt)] = a.n_sink + i * 32 + lane;
            if (sel_copy) sel_copy[prefix + __popc(mask & lt)] = a.n_sink + i * 32 + lane;
        }
        prefix += __popc(mask);
    }
    const int tail0 = a.NF - a.n_recent - a.n_cur;
    for (int t = lane; t < a.n_recent + a.n_cur; t += 32) {
        out[a.n_sink + kf + t] = tail0 + t;
        if (sel_copy) sel_copy[a.n_sink + kf + t] = tail0 + t;
    }
}

template <int D, int KPL>
__global__ void __launch_bounds__(SEL_THREADS) select_frames_kernel(const SelectFramesArgs a)
{
    constexpr int EPL = D / 32;
    const int lane = threadIdx.x & 31;
    const long long row = static_cast<long long>(blockIdx.x) * SEL_WARPS + (threadIdx.x >> 5);
    if (row >= static_cast<long long>(a.BH) * a.Rq) return;
    float qv[EPL];
    load_lane<EPL>(qv, a.q_pool + row * D + lane * EPL);
    frames_of_row<D, KPL>(a, row, lane, qv, a.frame_sel + row * a.n_sel, nullptr);
}

// The top-k_b blocks of selected frame slot s (frame tau) of scored row `row` (one
// warp), written ascending into the row's list at s * k_b. KPL = ceil(bpf / 32).
template <int D, int KPL>
__device__ __forceinline__ void blocks_of_frame(const SelectBlocksArgs& a, long long row, int s, int tau, int lane,
                                                const float (&qv)[D / 32])
{
    const int bh = static_cast<int>(row / a.Rq);
    int* out = a.block_list + row * a.list_cap + static_cast<long long>(s) * a.kb;
    if (s == 0 && lane == 0) a.block_count[row] = a.n_sel * a.kb;
    if (tau < 0 || tau >= a.NF) {
        // A frame id outside the call: write ids the attention kernel rejects.
        for (int t = lane; t < a.kb; t += 32) out[t] = -1;
        if (lane == 0) record_error(a.err, DEVERR_LIST | 3);
        return;
    }
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

// One warp per (row, selected-frame slot).
template <int D, int KPL>
__global__ void __launch_bounds__(SEL_THREADS) select_blocks_kernel(const SelectBlocksArgs a)
{
    constexpr int EPL = D / 32;
    const int lane = threadIdx.x & 31;
    const long long gw = static_cast<long long>(blockIdx.x) * SEL_WARPS + (threadIdx.x >> 5);
    if (gw >= static_cast<long long>(a.BH) * a.Rq * a.n_sel) return;
    const long long row = gw / a.n_sel;
    const int s = static_cast<int>(gw - row * a.n_sel);
    const int tau = (a.chunk_index == 1) ? s : __ldg(a.frame_sel + row * a.n_sel + s);
    float qv[EPL];
    load_lane<EPL>(qv, a.q_pool + row * D + lane * EPL);
    blocks_of_frame<D, KPL>(a, row, s, tau, lane, qv);
}

// Both levels for one scored row per CTA, in one launch: warp 0 picks T_r (to frame_sel
// and to shared memory), then warp w takes the blocks of selected frames w, w + W, ...
// The arithmetic is the two kernels' above, so the result is bit-identical to
// select_frames_kernel followed by select_blocks_kernel; the second launch and its
// dependent gap are gone.
template <int D, int KPLF, int KPLB>
__global__ void __launch_bounds__(SEL_FUSED_MAX_WARPS * 32) select_fused_kernel(const SelectFramesArgs fa,
                                                                                const SelectBlocksArgs ba)
{
    constexpr int EPL = D / 32;
    extern __shared__ int sel_s[];  // [n_sel]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, n_warps = blockDim.x >> 5;
    const long long row = blockIdx.x;
    float qv[EPL];
    load_lane<EPL>(qv, fa.q_pool + row * D + lane * EPL);
    if (warp == 0) frames_of_row<D, KPLF>(fa, row, lane, qv, fa.frame_sel + row * fa.n_sel, sel_s);
    __syncthreads();
    for (int s = warp; s < ba.n_sel; s += n_warps) blocks_of_frame<D, KPLB>(ba, row, s, sel_s[s], lane, qv);
}

// One-dimensional selection (the single-granularity variant of the ablation in
// "南洋理工大学打造视频生成新引擎", 163.com, section 4): every KV block of the head is a
// candidate. One CTA per scored row. A producer warp streams the head's pooled keys in
// groups of 32 candidates (16 KB at head_dim 128) into a 4-slot shared-memory ring with
// 1-D bulk copies; consumer warp w owns slot w and scores groups w, w + 4, ... into
// 32-bit orderable scores in shared memory, so each slot's uses are waited for in order
// by one warp. The four consumer warps then find the exact score T of the kb-th largest
// bit by bit from the top (32 rounds: per-thread counts, one warp reduction, the four
// warp counts through shared memory, one barrier per round) and write, in index order,
// every candidate scoring above T and the lowest-indexed ones scoring exactly T until kb
// are kept: the order of the two-level kernels' 64-bit keys (score, then lower index),
// so the list is that of a full sort.
constexpr int SEL1D_CONSUMERS = 4;
constexpr int SEL1D_THREADS = 32 * (SEL1D_CONSUMERS + 1);
constexpr int SEL1D_CT = 32 * SEL1D_CONSUMERS;  // consumer threads

template <int D>
constexpr size_t sel1d_ring_bytes()
{
    return static_cast<size_t>(SEL1D_CONSUMERS) * 32u * D * sizeof(float);
}

template <int D>
__global__ void __launch_bounds__(SEL1D_THREADS) select_blocks_1d_kernel(const SelectBlocks1dArgs a)
{
    constexpr int EPL = D / 32;
    constexpr int GROUP_FLOATS = 32 * D;
    extern __shared__ __align__(128) uint8_t sm1d[];
    float* ring = reinterpret_cast<float*>(sm1d);                                // [SEL1D_CONSUMERS][32][D]
    uint32_t* sc = reinterpret_cast<uint32_t*>(sm1d + sel1d_ring_bytes<D>());    // [Nkv]
    __shared__ uint64_t full[SEL1D_CONSUMERS], empty[SEL1D_CONSUMERS];
    __shared__ int wc[2][2][SEL1D_CONSUMERS];  // per-warp counts, double-buffered by round parity
    __shared__ int abort_word;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const long long row = blockIdx.x;
    const int n = a.Nkv;
    const int bh = static_cast<int>(row / a.Rq);
    int* out = a.block_list + row * a.list_cap;
    const int keep = (a.chunk_index == 1 || a.kb >= n) ? n : a.kb;
    if (threadIdx.x == 0) a.block_count[row] = keep;
    if (keep == n) {
        for (int g = threadIdx.x; g < n; g += SEL1D_THREADS) out[g] = g;
        return;
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < SEL1D_CONSUMERS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        abort_word = 0;
        fence_mbar_init();
    }
    __syncthreads();
    volatile int* abort_flag = &abort_word;
    const float* kblk = a.k_pool + static_cast<long long>(bh) * n * D;
    const int n_groups = (n + 31) / 32;
    if (warp == SEL1D_CONSUMERS) {
        // ---------------------------------------------------------------- producer
        int g = 0;
        for (; g < n_groups; ++g) {
            const int s = g % SEL1D_CONSUMERS;
            if (!mbar_wait(&empty[s], static_cast<uint32_t>(((g / SEL1D_CONSUMERS) & 1) ^ 1), abort_flag, a.err, 0x50))
                break;
            const uint32_t bytes = static_cast<uint32_t>(min(32, n - 32 * g)) * D * sizeof(float);
            mbar_arrive_expect_tx_elect(&full[s], bytes);
            bulk_load_elect(ring + s * GROUP_FLOATS, kblk + static_cast<long long>(g) * GROUP_FLOATS, bytes, &full[s]);
        }
        if (g < n_groups)  // aborted: let the copies already issued land before the CTA exits
            for (int g2 = max(0, g - SEL1D_CONSUMERS); g2 < g; ++g2)
                mbar_drain(&full[g2 % SEL1D_CONSUMERS], static_cast<uint32_t>((g2 / SEL1D_CONSUMERS) & 1), 10000000ull);
        return;
    }
    // -------------------------------------------------------------------- consumers
    float qv[EPL];
    load_lane<EPL>(qv, a.q_pool + row * D + lane * EPL);
    for (int g = warp; g < n_groups; g += SEL1D_CONSUMERS) {
        if (!mbar_wait(&full[warp], static_cast<uint32_t>((g / SEL1D_CONSUMERS) & 1), abort_flag, a.err, 0x51)) break;
        const int cnt = min(32, n - 32 * g);
        const float s = score_group<D, true>(qv, ring + warp * GROUP_FLOATS, 0, cnt, lane);
        if (lane < cnt) sc[32 * g + lane] = orderable(s);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[warp]);
    }
    // scores complete (or the CTA gave up: the same decision in every consumer thread)
    if (named_bar_or(1, SEL1D_CT, *abort_flag != 0)) return;
    const int tid = threadIdx.x;
    // T = the largest 32-bit value with at least `keep` scores >= T, built bit by bit.
    // Round `bit` writes wc[bit & 1][0]; a buffer is rewritten two rounds later, after
    // every consumer thread has passed the barrier of the round in between.
    uint32_t prefix = 0;
    for (int bit = 31; bit >= 0; --bit) {
        const uint32_t cand = prefix | (1u << bit);
        int c = 0;
        for (int g = tid; g < n; g += SEL1D_CT) c += sc[g] >= cand ? 1 : 0;
        c = __reduce_add_sync(0xffffffffu, c);
        if (lane == 0) wc[bit & 1][0][warp] = c;
        named_bar_sync(1, SEL1D_CT);
        int tot = 0;
#pragma unroll
        for (int w = 0; w < SEL1D_CONSUMERS; ++w) tot += wc[bit & 1][0][w];
        if (tot >= keep) prefix = cand;
    }
    int above = 0;
    {
        int c = 0;
        for (int g = tid; g < n; g += SEL1D_CT) c += sc[g] > prefix ? 1 : 0;
        c = __reduce_add_sync(0xffffffffu, c);
        if (lane == 0) wc[1][1][warp] = c;  // not used by the rounds above
        named_bar_sync(1, SEL1D_CT);
#pragma unroll
        for (int w = 0; w < SEL1D_CONSUMERS; ++w) above += wc[1][1][w];
    }
    const int need = keep - above;  // scores equal to T still to take, lowest index first
    // Index-order compaction, SEL1D_CT candidates per chunk. Before candidate g: gt_before
    // scores above T and eq_before equal to T; g goes to gt_before + min(eq_before, need).
    const uint32_t lt = (1u << lane) - 1u;
    int gt_base = 0, eq_base = 0;
    for (int c0 = 0, it = 0; c0 < n; c0 += SEL1D_CT, ++it) {
        const int g = c0 + tid;
        const uint32_t v = g < n ? sc[g] : 0u;
        const bool gt = g < n && v > prefix;
        const bool eq = g < n && v == prefix;
        const uint32_t gm = __ballot_sync(0xffffffffu, gt);
        const uint32_t em = __ballot_sync(0xffffffffu, eq);
        const int b = it & 1;
        if (lane == 0) {
            wc[b][0][warp] = __popc(gm);
            wc[b][1][warp] = __popc(em);
        }
        named_bar_sync(1, SEL1D_CT);
        int pg = 0, pe = 0, tg = 0, te = 0;
#pragma unroll
        for (int w = 0; w < SEL1D_CONSUMERS; ++w) {
            const int x = wc[b][0][w], y = wc[b][1][w];
            pg += w < warp ? x : 0;
            pe += w < warp ? y : 0;
            tg += x;
            te += y;
        }
        const int gt_before = gt_base + pg + __popc(gm & lt);
        const int eq_before = eq_base + pe + __popc(em & lt);
        if (gt || (eq && eq_before < need)) out[gt_before + min(eq_before, need)] = g;
        gt_base += tg;
        eq_base += te;
    }
}

template <int D>
cudaError_t launch_blocks_1d_d(const SelectBlocks1dArgs& a, cudaStream_t s)
{
    const size_t smem = sel1d_ring_bytes<D>() + static_cast<size_t>(a.Nkv) * sizeof(uint32_t);
    static int configured_device = -1;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (configured_device != dev) {
        e = cudaFuncSetAttribute(select_blocks_1d_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(sel1d_ring_bytes<D>() + SEL1D_MAX_NKV * sizeof(uint32_t)));
        if (e != cudaSuccess) return e;
        configured_device = dev;
    }
    const unsigned grid = static_cast<unsigned>(static_cast<long long>(a.BH) * a.Rq);
    select_blocks_1d_kernel<D><<<grid, SEL1D_THREADS, smem, s>>>(a);
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

template <int D, int KPLF, int KPLB>
cudaError_t launch_fused_k(const SelectFramesArgs& fa, const SelectBlocksArgs& ba, cudaStream_t s)
{
    const unsigned grid = static_cast<unsigned>(static_cast<long long>(fa.BH) * fa.Rq);
    const int warps = ba.n_sel < SEL_FUSED_MAX_WARPS ? ba.n_sel : SEL_FUSED_MAX_WARPS;
    select_fused_kernel<D, KPLF, KPLB><<<grid, 32 * warps, static_cast<size_t>(fa.n_sel) * sizeof(int), s>>>(fa, ba);
    return cudaGetLastError();
}

template <int D, int KPLF>
cudaError_t launch_fused_b(const SelectFramesArgs& fa, const SelectBlocksArgs& ba, cudaStream_t s)
{
    const int kpl = (ba.bpf + 31) / 32;
    if (kpl <= 1) return launch_fused_k<D, KPLF, 1>(fa, ba, s);
    if (kpl <= 2) return launch_fused_k<D, KPLF, 2>(fa, ba, s);
    return launch_fused_k<D, KPLF, 4>(fa, ba, s);
}

template <int D>
cudaError_t launch_fused_d(const SelectFramesArgs& fa, const SelectBlocksArgs& ba, cudaStream_t s)
{
    const int n_mem = fa.NF - fa.n_sink - fa.n_recent - fa.n_cur;
    const int kpl = (n_mem + 31) / 32;
    if (fa.chunk_index == 1 || kpl <= 1) return launch_fused_b<D, 1>(fa, ba, s);
    if (kpl <= 2) return launch_fused_b<D, 2>(fa, ba, s);
    if (kpl <= 4) return launch_fused_b<D, 4>(fa, ba, s);
    if (kpl <= 8) return launch_fused_b<D, 8>(fa, ba, s);
    if (kpl <= 16) return launch_fused_b<D, 16>(fa, ba, s);
    return launch_fused_b<D, 32>(fa, ba, s);
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

cudaError_t launch_select_fused(const SelectFramesArgs& fa, const SelectBlocksArgs& ba, cudaStream_t s)
{
    if (static_cast<long long>(fa.BH) * fa.Rq <= 0) return cudaSuccess;
    return fa.D == 128 ? launch_fused_d<128>(fa, ba, s) : launch_fused_d<64>(fa, ba, s);
}

cudaError_t launch_select_blocks(const SelectBlocksArgs& a, cudaStream_t s)
{
    const long long warps = static_cast<long long>(a.BH) * a.Rq * a.n_sel;
    if (warps <= 0) return cudaSuccess;
    const unsigned grid = static_cast<unsigned>((warps + SEL_WARPS - 1) / SEL_WARPS);
    return a.D == 128 ? launch_blocks_d<128>(a, grid, s) : launch_blocks_d<64>(a, grid, s);
}

}  // namespace lf
