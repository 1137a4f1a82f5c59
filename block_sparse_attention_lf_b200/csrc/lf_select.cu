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
// Both levels run in one launch (select_fused_kernel, one CTA per scored row). The
// one-dimensional variant (global block top-k, no frame level) scores tiles of rows
// of one head through a bulk-copy ring (select_1d_tile_kernel), or one row per CTA for
// heads of more than 2,048 blocks (select_blocks_1d_kernel).
#include "lf_device.cuh"
#include "lf_internal.h"
#include "lf_score.cuh"

namespace lf {
namespace {

constexpr int SEL_THREADS = 256;
constexpr int SEL_WARPS = SEL_THREADS / 32;
constexpr int SEL_FUSED_MAX_WARPS = 16;
// warps per fused-selection CTA: few warps keep every row's CTA resident at once (900 rows
// at 6-7 CTAs per SM). With the forced slots scored beside the frame level, 4 warps took
// 18.4 / 20.5 / 29.6 us at layer480p / longvideo480p / patterns480p against 20.5 / 22.5 /
// 32.8 us for 3 warps and 22.5 / 26.6 / 30.7 us for 5 (the frame level first, then all
// slots, on 3 warps: 18.5 / 24.6 / 32.8 us); one warp per selected frame (9) was slower still.
constexpr int SEL_FUSED_WARPS = 4;

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

// The top-k_b of a frame's block keys (key slot i of lane l = block i * 32 + l, 0 = none) by
// rank counting (rank = number of larger keys), written ascending by a ballot compaction.
template <int KPL>
__device__ __forceinline__ void write_top_blocks(const SelectBlocksArgs& a, int* out, const uint64_t (&key)[KPL],
                                                 int tau, int lane)
{
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

    write_top_blocks<KPL>(a, out, key, tau, lane);
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

// Both levels for one scored row per CTA, in one launch. The forced frames' slots of T_r
// (sinks, recent and current frames) are known before the frame level, so while warp 0
// picks T_r (to frame_sel and to shared memory) the other warps already take the block
// top-k of those slots; the selected memory frames' slots follow once warp 0 has published
// them (barrier 1: warp 0 arrives, every other warp syncs once). Slots are handed out in
// that order from a shared counter. The arithmetic is the two kernels' above, so the result
// is bit-identical to select_frames_kernel followed by select_blocks_kernel.
template <int D, int KPLF, int KPLB>
__global__ void __launch_bounds__(SEL_FUSED_MAX_WARPS * 32) select_fused_kernel(const SelectFramesArgs fa,
                                                                                const SelectBlocksArgs ba)
{
    constexpr int EPL = D / 32;
    extern __shared__ int sel_s[];  // [n_sel]
    __shared__ int next_slot;
    // a programmatic dependent of the pooling: wait for its outputs, and let the attention
    // that follows be scheduled early (it waits for this grid the same way)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (threadIdx.x == 0) {
        asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
        next_slot = 0;
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, n_warps = blockDim.x >> 5;
    const long long row = blockIdx.x;
    float qv[EPL];
    load_lane<EPL>(qv, fa.q_pool + row * D + lane * EPL);
    // items [0, n_forced) are the forced slots in slot order, then the kf selected ones
    int kf = 0;
    if (fa.chunk_index != 1) {
        const int n_mem = fa.NF - fa.n_sink - fa.n_recent - fa.n_cur;
        kf = fa.topk < n_mem ? fa.topk : n_mem;
    }
    const int n_forced = ba.n_sel - kf;
    const int tail0 = fa.NF - fa.n_recent - fa.n_cur;
    const int bar_threads = 32 * n_warps;
    __syncthreads();  // next_slot is initialised
    bool synced = true;
    if (warp == 0) {
        frames_of_row<D, KPLF>(fa, row, lane, qv, fa.frame_sel + row * fa.n_sel, sel_s);
        __syncwarp();
        if (n_warps > 1) named_bar_arrive(1, bar_threads);
    } else {
        synced = false;
    }
    for (;;) {
        int it = 0;
        if (lane == 0) it = atomicAdd(&next_slot, 1);
        it = __shfl_sync(0xffffffffu, it, 0);
        if (it >= ba.n_sel) break;
        int s, tau;
        if (it < n_forced) {
            s = it < fa.n_sink ? it : it + kf;
            tau = (fa.chunk_index == 1 || s < fa.n_sink) ? s : tail0 + (s - fa.n_sink - kf);
        } else {
            if (!synced) {
                named_bar_sync(1, bar_threads);
                synced = true;
            }
            s = fa.n_sink + (it - n_forced);
            tau = sel_s[s];
        }
        blocks_of_frame<D, KPLB>(ba, row, s, tau, lane, qv);
    }
    if (!synced) named_bar_sync(1, bar_threads);
}

// ---- one-dimensional selection, tiled, through a bulk-copy ring ----------------------
// One CTA per tile of TR_ROWS scored rows (query blocks) of one head. A producer warp
// streams the head's pooled keys in groups of 32 candidates (16 KB at head_dim 128) into a
// shared-memory ring with 1-D bulk copies, so each pooled key crosses L2 -> SM once per tile
// instead of once per row. CONS consumer warps form CONS / 4 classes of four; warp w scores
// rows 2(w % 4) and 2(w % 4) + 1 against the groups g with g % (CONS / 4) == w / 4: each
// candidate slice read from shared memory feeds two inner products, and the classes work on
// different groups at once (the scoring is latency-bound: 16 warps score a tile about twice
// as fast as 8). The ring has CONS / 2 slots, two per class; slot s only ever holds groups of
// class s % (CONS / 4) and is consumed by the same four warps, in order. Groups are laid out
// as in the one-row kernel (32 consecutive blocks from the head's first), so every score, and
// with it every list, is bit-identical to its. (The two-level selection tiled the same way,
// all of a head's blocks scored per tile, ran at 34.8 us against 23.6 us for
// select_fused_kernel, which scores only the selected frames' blocks; it was not kept.)
constexpr int TR_ROWS = 8;
constexpr int TR_1D_MAX_NKV = 2048;  // scores of a row in registers (64 per lane); beyond: the one-row kernel

template <int D, int CONS>
constexpr size_t tr_ring_bytes()
{
    return static_cast<size_t>(CONS / 2) * 32u * D * sizeof(float);
}

template <int CONS>
struct TileRing {
    static constexpr int SLOTS = CONS / 2;
    uint64_t full[SLOTS], empty[SLOTS];
    int abort;
};

// Groups of 32 consecutive candidates of the head (the last one may be shorter).
struct TileGroups {
    int n, n_groups;
    __device__ __forceinline__ explicit TileGroups(int n_) : n(n_), n_groups((n_ + 31) / 32) {}
    __device__ __forceinline__ int base(int g) const { return 32 * g; }
    __device__ __forceinline__ int count(int g) const { return min(32, n - 32 * g); }
};

// The two-row scoring of score_group (SHARED: rows in shared memory).
template <int D, bool SHARED>
__device__ __forceinline__ void score_group2(const float (&q0)[D / 32], const float (&q1)[D / 32], const float* rows,
                                             int n, int lane, float& s0, float& s1)
{
    constexpr int EPL = D / 32;
    float p0[32], p1[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) {
        p0[c] = 0.f;
        p1[c] = 0.f;
        if (c < n) {
            float kv[EPL];
            load_lane<EPL, SHARED>(kv, rows + static_cast<long long>(c) * D + lane * EPL);
#pragma unroll
            for (int e = 0; e < EPL; ++e) {
                p0[c] = fmaf(q0[e], kv[e], p0[c]);
                p1[c] = fmaf(q1[e], kv[e], p1[c]);
            }
        }
    }
    transpose_reduce_sum(p0, lane);
    transpose_reduce_sum(p1, lane);
    s0 = p0[0];
    s1 = p1[0];
}

template <int CONS>
__device__ __forceinline__ void tile_ring_init(TileRing<CONS>& r)
{
    for (int s = 0; s < TileRing<CONS>::SLOTS; ++s) {
        mbar_init(&r.full[s], 1);
        mbar_init(&r.empty[s], 4);  // the four warps of the slot's class
    }
    r.abort = 0;
    fence_mbar_init();
}

// Producer warp: every group of the head, in order.
template <int D, int CONS>
__device__ __forceinline__ void tile_produce(TileRing<CONS>& r, const TileGroups& tg, const float* kblk, float* ring,
                                             int* err)
{
    constexpr int TR_SLOTS = TileRing<CONS>::SLOTS;
    volatile int* abort_flag = &r.abort;
    int g = 0;
    for (; g < tg.n_groups; ++g) {
        const int s = g % TR_SLOTS;
        if (!mbar_wait(&r.empty[s], static_cast<uint32_t>(((g / TR_SLOTS) & 1) ^ 1), abort_flag, err, 0x52)) break;
        const uint32_t bytes = static_cast<uint32_t>(tg.count(g)) * D * sizeof(float);
        mbar_arrive_expect_tx_elect(&r.full[s], bytes);
        bulk_load_elect(ring + s * 32 * D, kblk + static_cast<long long>(tg.base(g)) * D, bytes, &r.full[s]);
    }
    if (g < tg.n_groups)  // aborted: let the copies already issued land before the CTA exits
        for (int g2 = max(0, g - TR_SLOTS); g2 < g; ++g2)
            mbar_drain(&r.full[g2 % TR_SLOTS], static_cast<uint32_t>((g2 / TR_SLOTS) & 1), 10000000ull);
}

// Consumer warps: the tile's scores into sc[TR_ROWS][n]; rows past rows_valid score with a
// zero query and are never read. Returns false when the CTA gave up; the answer is the same
// in every consumer thread, and the call is the barrier after which sc is complete.
template <int D, int CONS>
__device__ __forceinline__ bool tile_score(TileRing<CONS>& r, const TileGroups& tg, const float* q_pool, long long row0,
                                           int rows_valid, int n, const float* ring, float* sc, int* err, int warp,
                                           int lane)
{
    constexpr int EPL = D / 32;
    constexpr int TR_SLOTS = TileRing<CONS>::SLOTS;
    volatile int* abort_flag = &r.abort;
    const int ra = 2 * (warp & 3), rb = ra + 1, par = warp >> 2;
    float q0[EPL], q1[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
        q0[e] = 0.f;
        q1[e] = 0.f;
    }
    if (ra < rows_valid) load_lane<EPL>(q0, q_pool + (row0 + ra) * D + lane * EPL);
    if (rb < rows_valid) load_lane<EPL>(q1, q_pool + (row0 + rb) * D + lane * EPL);
    for (int g = par; g < tg.n_groups; g += CONS / 4) {
        const int s = g % TR_SLOTS;
        if (!mbar_wait(&r.full[s], static_cast<uint32_t>((g / TR_SLOTS) & 1), abort_flag, err, 0x53)) break;
        const int base = tg.base(g), cnt = tg.count(g);
        float s0, s1;
        score_group2<D, true>(q0, q1, ring + s * 32 * D, cnt, lane, s0, s1);
        if (lane < cnt) {
            sc[ra * n + base + lane] = s0;
            sc[rb * n + base + lane] = s1;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&r.empty[s]);
    }
    return !named_bar_or(1, 32 * CONS, *abort_flag != 0);
}

// One-dimensional selection over the tile's scores: each warp its row, the row's scores in
// registers (VPL per lane, candidate 32 i + lane in slot i); the threshold score T of the
// kept count is built bit by bit (32 rounds of per-lane counts and one warp reduction), then
// every candidate above T and the lowest-indexed ones equal to T are written in index order.
template <int D, int VPL, int CONS>
__global__ void __launch_bounds__(32 * CONS + 32) select_1d_tile_kernel(const SelectBlocks1dArgs a)
{
    extern __shared__ __align__(128) uint8_t tr_smem[];
    __shared__ TileRing<CONS> rc;
    const int n = a.Nkv;
    float* ring = reinterpret_cast<float*>(tr_smem);
    float* sc = reinterpret_cast<float*>(tr_smem + tr_ring_bytes<D, CONS>());  // [TR_ROWS][n]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int tiles = (a.Rq + TR_ROWS - 1) / TR_ROWS;
    const int bh = static_cast<int>(blockIdx.x / tiles);
    const int r_in = static_cast<int>(blockIdx.x - static_cast<long long>(bh) * tiles) * TR_ROWS;
    const int rows_valid = min(TR_ROWS, a.Rq - r_in);
    const long long row0 = static_cast<long long>(bh) * a.Rq + r_in;
    const int keep = (a.chunk_index == 1 || a.kb >= n) ? n : a.kb;
    if (keep == n) {
        if (warp < rows_valid) {
            int* out = a.block_list + (row0 + warp) * a.list_cap;
            if (lane == 0) a.block_count[row0 + warp] = keep;
            for (int g = lane; g < n; g += 32) out[g] = g;
        }
        return;
    }
    const TileGroups tg(n);
    if (threadIdx.x == 0) tile_ring_init(rc);
    __syncthreads();
    if (warp == CONS) {
        tile_produce<D, CONS>(rc, tg, a.k_pool + static_cast<long long>(bh) * n * D, ring, a.err);
        return;
    }
    if (!tile_score<D, CONS>(rc, tg, a.q_pool, row0, rows_valid, n, ring, sc, a.err, warp, lane)) return;
    if (warp >= rows_valid) return;
    const long long row = row0 + warp;
    int* out = a.block_list + row * a.list_cap;
    if (lane == 0) a.block_count[row] = keep;
    uint32_t v[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const int g = 32 * i + lane;
        v[i] = g < n ? orderable(sc[warp * n + g]) : 0u;
    }
    uint32_t prefix = 0;
    for (int bit = 31; bit >= 0; --bit) {
        const uint32_t cand = prefix | (1u << bit);
        int c = 0;
#pragma unroll
        for (int i = 0; i < VPL; ++i) c += (32 * i + lane < n && v[i] >= cand) ? 1 : 0;
        if (__reduce_add_sync(0xffffffffu, c) >= keep) prefix = cand;
    }
    int above = 0;
#pragma unroll
    for (int i = 0; i < VPL; ++i) above += (32 * i + lane < n && v[i] > prefix) ? 1 : 0;
    const int need = keep - __reduce_add_sync(0xffffffffu, above);  // scores equal to T still to take
    int pos = 0, eq_seen = 0;
    const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        const int g = 32 * i + lane;
        const bool valid = g < n;
        const bool eq = valid && v[i] == prefix;
        const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
        const bool take = (valid && v[i] > prefix) || (eq && eq_seen + __popc(eqm & lt) < need);
        const uint32_t tm = __ballot_sync(0xffffffffu, take);
        if (take) out[pos + __popc(tm & lt)] = g;
        pos += __popc(tm);
        eq_seen += __popc(eqm);
    }
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

// Shared-memory opt-in of a tiled kernel, once per device.
template <typename Kernel>
cudaError_t tile_smem_optin(Kernel k, int& configured_device, size_t bytes)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (configured_device != dev) {
        e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
        if (e != cudaSuccess) return e;
        configured_device = dev;
    }
    return cudaSuccess;
}

template <int D, int VPL, int CONS>
cudaError_t launch_1d_tile_c(const SelectBlocks1dArgs& a, long long grid, cudaStream_t s)
{
    static int configured_device = -1;
    cudaError_t e = tile_smem_optin(select_1d_tile_kernel<D, VPL, CONS>, configured_device,
                                    tr_ring_bytes<D, CONS>() + TR_ROWS * TR_1D_MAX_NKV * sizeof(float));
    if (e != cudaSuccess) return e;
    select_1d_tile_kernel<D, VPL, CONS><<<static_cast<unsigned>(grid), 32 * CONS + 32,
                                          tr_ring_bytes<D, CONS>() + static_cast<size_t>(TR_ROWS) * a.Nkv * sizeof(float),
                                          s>>>(a);
    return cudaGetLastError();
}

// 16 consumer warps (a 128 KB ring at head_dim 128, one CTA per SM) when the tiles fit in one
// wave; otherwise 8 (a 64 KB ring, two CTAs per SM).
template <int D, int VPL>
cudaError_t launch_1d_tile(const SelectBlocks1dArgs& a, cudaStream_t s)
{
    const long long grid = static_cast<long long>(a.BH) * ((a.Rq + TR_ROWS - 1) / TR_ROWS);
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    if (grid <= sms) return launch_1d_tile_c<D, VPL, 16>(a, grid, s);
    return launch_1d_tile_c<D, VPL, 8>(a, grid, s);
}

template <int D>
cudaError_t launch_blocks_1d_d(const SelectBlocks1dArgs& a, cudaStream_t s)
{
    if (a.Nkv <= TR_1D_MAX_NKV) {
        const int vpl = (a.Nkv + 31) / 32;
        if (vpl <= 4) return launch_1d_tile<D, 4>(a, s);
        if (vpl <= 8) return launch_1d_tile<D, 8>(a, s);
        if (vpl <= 16) return launch_1d_tile<D, 16>(a, s);
        if (vpl <= 20) return launch_1d_tile<D, 20>(a, s);
        if (vpl <= 24) return launch_1d_tile<D, 24>(a, s);
        if (vpl <= 32) return launch_1d_tile<D, 32>(a, s);
        if (vpl <= 48) return launch_1d_tile<D, 48>(a, s);
        return launch_1d_tile<D, 64>(a, s);
    }
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
    const int warps = ba.n_sel < SEL_FUSED_WARPS ? ba.n_sel : SEL_FUSED_WARPS;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(32 * warps);
    cfg.dynamicSmemBytes = static_cast<size_t>(fa.n_sel) * sizeof(int);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see select_fused_kernel
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, select_fused_kernel<D, KPLF, KPLB>, fa, ba);
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
