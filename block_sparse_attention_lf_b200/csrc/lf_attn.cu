// lf_attn.cu -- block-sparse softmax attention of one HSA call on sm_100a
// tensor cores ("Light Forcing：通过稀疏注意力加速自回归视频扩散",
// paper.rainbus.top, execution flow, stage 3, final step: attention computed
// only over the kept (frame, block) pairs of B_r).
//
// Design (B200-first; the pages' kernel is prior art only):
//   * One CTA per query block (64 query tokens of one head, its own KV block
//     list). CTAs are ordered head-major so a head's K/V stay L2-resident while
//     its query blocks run.
//   * KV-major formulation. A tile is two listed KV blocks (128 tokens). The
//     tensor core computes S^T = K_tile * Q^T (M = 128 KV tokens, N = 64
//     queries, K = head_dim) into TMEM, and O^T += V_tile^T * P^T (M = 128
//     head-dim rows, N = 64 queries, K = 128 KV tokens). Both MMAs run with
//     M = 128 (M = 64 issues at half rate on this part) on exactly the listed
//     blocks, with no union of neighbouring query blocks' lists.
//   * Gather. K and V dominate the traffic (each query block reads its own
//     ~100 blocks from L2). Small TMA boxes cap the per-SM L2 bandwidth, so
//     for head_dim 128 each 64-token block (16 KB, contiguous) arrives as ONE
//     4-D box {64 elems, 8 rows, 2 panels, 8 row groups} that lands in an
//     interleaved layout [row group][panel][8 rows x 128 B] (128-byte swizzle).
//     Its 8-row groups sit a uniform 2 KB apart, so one smem descriptor spans
//     both blocks of a tile for the S^T MMA (SBO = 2 KB, panel at +1 KB) and
//     for the PV MMA (MN-major: LBO = 1 KB between head-dim panels, SBO = 2 KB
//     between 8-row groups). Frames whose token count is not a multiple of 8,
//     and head_dim 64, use 2-D boxes per 64-wide panel into a plain
//     [panel][row] layout instead.
//   * Warp roles (384 threads): warp 0 issues the Q and K loads, warp 1 the V
//     loads (so a V slot that is still in use never delays K prefetch), warp 2
//     allocates TMEM and issues tcgen05.mma from one thread, warp 3 idles,
//     warps 4-11 are two softmax warpgroups. TMEM lane t of S^T is KV token t
//     of the tile, so each softmax thread owns one KV token of a tile and all
//     64 query columns.
//   * Ping-pong. Warpgroup g takes the tiles i with i % 2 == g, with its own
//     running maxima, its own O^T accumulator in TMEM and its own P buffer, so
//     one warpgroup exponentiates while the other waits for its next scores;
//     the two partial softmaxes are merged once in the epilogue
//     (O = (O_0 2^(m_0-M) + O_1 2^(m_1-M)) / (l_0 2^(m_0-M) + l_1 2^(m_1-M))).
//   * Online softmax in fp32, base 2, with a lazy stabiliser: each query
//     column keeps m (running max of scale*log2(e)*score, in shared memory); a
//     tile whose scores stay within m + 8 (p <= 256) is exponentiated against
//     the current m with no cross-thread work; only when some score exceeds
//     that bound does the warpgroup compute the exact column maxima of the tile
//     (butterfly reductions + shared memory) and rescale its O^T columns in
//     TMEM. Row sums are kept per thread and reduced once at the end.
//   * P^T goes to shared memory as bf16 in the 128-byte-swizzled MN-major
//     layout the MMA reads; masked KV tokens (past the end of a partial block,
//     or the unused half of an odd last tile) get P = 0.
//   * Pipelines: K ring of 3 slots, V ring of 2, four S buffers in TMEM (S is
//     issued up to four tiles ahead), one P buffer per warpgroup. The MMA
//     thread never blocks on one operand while another MMA is ready: it polls
//     its barriers and issues whichever PV (first) or S is ready.
//   * Every mbarrier wait is bounded (1 s); on expiry the CTA sets an abort
//     flag and the device error word, every role runs its remaining steps
//     without waiting, in-flight copies and MMAs are drained, TMEM is freed,
//     and the kernel returns.
#include "lf_device.cuh"
#include "lf_internal.h"

#include <cuda_bf16.h>

#include <cstddef>

namespace lf {
namespace {

constexpr int ATTN_THREADS = 384;
constexpr int W_KPROD = 0, W_VPROD = 1, W_MMA = 2, W_SOFT0 = 4;
constexpr int KSLOTS = 3;
constexpr int VSLOTS = 2;
constexpr float LAZY_RESCALE_LOG2 = 8.0f;  // p may reach 2^8 before the stabiliser moves
constexpr uint32_t TMEM_COLS = 512;         // S buffers 0-3: columns 64*b; O^T of warpgroup g: 256 + 64*g
constexpr int ROWS_SMEM = 1024;             // list entries whose row counts are cached in smem

// Shared-memory plan. IL selects the interleaved K/V layout (head_dim 128,
// one 4-D box per block); otherwise K/V use [panel][128 rows x 128 B].
template <int D, bool IL>
struct AttnLayout {
    static constexpr int NP = D / 64;                  // 64-element panels of head_dim
    static constexpr uint32_t PANEL_Q = 64u * 128u;     // 64 rows x 128 B
    static constexpr uint32_t PANEL_KV = 128u * 128u;   // 128 rows x 128 B (panel layout)
    static constexpr uint32_t BLOCK_IL = 16384u;        // one 64 x 128 bf16 block (interleaved)
    static constexpr uint32_t Q_BYTES = NP * PANEL_Q;
    static constexpr uint32_t K_SLOT = NP * PANEL_KV;
    static constexpr uint32_t V_SLOT = 2u * PANEL_KV;   // the PV MMA has M = 128 head-dim rows
    static constexpr uint32_t P_BUF = 128u * 128u;      // P^T: 128 KV rows x 64 queries bf16
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
    static constexpr uint32_t OFF_V = OFF_K + KSLOTS * K_SLOT;
    static constexpr uint32_t OFF_P = OFF_V + VSLOTS * V_SLOT;
    static constexpr uint32_t OFF_AUX = OFF_P + 2u * P_BUF;
    // smem descriptor strides of the K/V tiles
    static constexpr uint32_t KV_SBO = IL ? 2048u : 1024u;          // between 8-row groups
    static constexpr uint32_t KV_PANEL = IL ? 1024u : PANEL_KV;     // between 64-wide panels
    static constexpr uint32_t KV_K16 = IL ? 4096u : 2048u;          // 16 KV rows (one PV k-step)
    static_assert(!IL || D == 128, "interleaved layout is for head_dim 128");
};

struct AttnAux {
    uint64_t q_full;
    uint64_t k_full[KSLOTS], k_empty[KSLOTS];
    uint64_t v_full[VSLOTS], v_empty[VSLOTS];
    uint64_t s_full[4], s_free[4], p_full[2], p_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    float red[2][4][64];
    float lsum[2][64];             // softmax denominators of each warpgroup's columns
    alignas(16) float m_s[2][64];  // running max (log2 units) per warpgroup and query column (read as float4)
    uint8_t rows[ROWS_SMEM];       // valid token rows of list entry b (0: not a valid block)
};

static_assert(offsetof(AttnAux, m_s) % 16 == 0, "m_s is read with 16-byte loads");

template <int D, bool IL>
constexpr uint32_t attn_smem_bytes()
{
    return AttnLayout<D, IL>::OFF_AUX + static_cast<uint32_t>(sizeof(AttnAux)) + 1024u;
}

template <bool MAX>
__device__ __forceinline__ void transpose_reduce(float (&v)[32], int lane)
{
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) {
        const bool upper = (lane & s) != 0;
#pragma unroll
        for (int i = 0; i < s; ++i) {
            const float send = upper ? v[i] : v[i + s];
            const float keep = upper ? v[i + s] : v[i];
            const float recv = __shfl_xor_sync(0xffffffffu, send, s);
            v[i] = MAX ? fmaxf(keep, recv) : keep + recv;
        }
    }
}

// Token rows of KV block g (0 when g is not a valid block id) and its first
// row in the flattened [B*H*kv_stride, D] view of k / v.
__device__ __forceinline__ int block_rows(const AttnArgs& a, int g, int bh, int* first_row)
{
    if (g < 0 || g >= a.Nkv) return 0;
    const int tau = g / a.bpf;
    const int j = g - tau * a.bpf;
    *first_row = static_cast<int>(static_cast<long long>(bh) * a.kv_stride + static_cast<long long>(tau) * a.F + j * 64);
    return (j == a.bpf - 1) ? a.rem : 64;
}

__device__ __forceinline__ void tma_load_4d(void* smem_dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                                            uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
        : "memory");
}

// Load one KV block (`rows` valid tokens starting at flattened row `first`)
// into half `h` of a K or V slot.
template <int D, bool IL>
__device__ __forceinline__ void load_block(uint8_t* slot, int h, int rows, int first, const CUtensorMap* full,
                                           const CUtensorMap* part, uint64_t* bar)
{
    using L = AttnLayout<D, IL>;
    const CUtensorMap* m = rows == 64 ? full : part;
    if constexpr (IL) {
        tma_load_4d(slot + h * L::BLOCK_IL, m, 0, 0, 0, first >> 3, bar);
    } else {
#pragma unroll
        for (int p = 0; p < L::NP; ++p) tma_load_2d(slot + p * L::PANEL_KV + h * 64 * 128, m, p * 64, first, bar);
    }
}

template <int D, bool IL>
__global__ void __launch_bounds__(ATTN_THREADS, 1)
attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_q_rem,
            const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_k_rem,
            const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_v_rem,
            const AttnArgs a)
{
    using L = AttnLayout<D, IL>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    AttnAux& x = *reinterpret_cast<AttnAux*>(smem + L::OFF_AUX);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int row = blockIdx.x;
    const int bh = row / a.Rq;
    const int r = row - bh * a.Rq;
    int cnt = __ldg(a.block_count + row);
    if (cnt < 0 || cnt > a.list_cap) {
        if (tid == 0) record_error(a.err, DEVERR_LIST | 1);
        cnt = cnt < 0 ? 0 : a.list_cap;
    }
    const int* lst = a.block_list + static_cast<long long>(row) * a.list_cap;
    const int n_tiles = (cnt + 1) >> 1;
    const int fq = r / a.bpf;
    const int jq = r - fq * a.bpf;
    const int q_rows = (jq == a.bpf - 1) ? a.rem : 64;
    const int q_row0 = bh * a.Lq + fq * a.F + jq * 64;

    if (tid == 0) {
        mbar_init(&x.q_full, 1);
        for (int s = 0; s < KSLOTS; ++s) { mbar_init(&x.k_full[s], 1); mbar_init(&x.k_empty[s], 1); }
        for (int s = 0; s < VSLOTS; ++s) { mbar_init(&x.v_full[s], 1); mbar_init(&x.v_empty[s], 1); }
        for (int s = 0; s < 4; ++s) {
            mbar_init(&x.s_full[s], 1);
            mbar_init(&x.s_free[s], 4);  // one arrival per warp of the owning warpgroup
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&x.p_full[s], 4);
            mbar_init(&x.p_empty[s], 1);
        }
        mbar_init(&x.drain, 1);
        x.abort = 0;
        fence_mbar_init();
    }
    if (warp == W_MMA) {
        tmem_alloc(&x.tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    if (tid < 128) x.m_s[tid >> 6][tid & 63] = -INFINITY;
    for (int b = tid; b < min(cnt, ROWS_SMEM); b += ATTN_THREADS) {
        int first;
        x.rows[b] = static_cast<uint8_t>(block_rows(a, __ldg(lst + b), bh, &first));
    }
    // V slots are read in full by the PV MMA (M = 128 head-dim rows, K = 128
    // KV rows) even where a tile loads fewer rows; they start at zero so those
    // rows are finite (P is zero there). Q rows past a partial query block
    // only feed discarded output columns; zero them as well.
    {
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        uint4* vz = reinterpret_cast<uint4*>(smem + L::OFF_V);
        for (int i = tid; i < static_cast<int>(VSLOTS * L::V_SLOT / 16); i += ATTN_THREADS) vz[i] = z;
        if (q_rows < 64) {
            uint4* qz = reinterpret_cast<uint4*>(smem + L::OFF_Q);
            for (int i = tid; i < static_cast<int>(L::Q_BYTES / 16); i += ATTN_THREADS) qz[i] = z;
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = x.tmem_base;
    volatile int* abort_flag = &x.abort;

    if (warp == W_KPROD || warp == W_VPROD) {
        // ------------------------------------------------------------ producers
        if (lane == 0) {
            const bool is_k = warp == W_KPROD;
            const int nslots = is_k ? KSLOTS : VSLOTS;
            uint64_t* full = is_k ? x.k_full : x.v_full;
            uint64_t* empty = is_k ? x.k_empty : x.v_empty;
            uint8_t* base = smem + (is_k ? L::OFF_K : L::OFF_V);
            const uint32_t slot_bytes = is_k ? L::K_SLOT : L::V_SLOT;
            const CUtensorMap* mfull = is_k ? &tm_k : &tm_v;
            const CUtensorMap* mpart = is_k ? &tm_k_rem : &tm_v_rem;
            tma_prefetch_desc(mfull);
            if (is_k) {
                const CUtensorMap* mq = (q_rows == 64) ? &tm_q : &tm_q_rem;
                mbar_arrive_expect_tx(&x.q_full, static_cast<uint32_t>(L::NP * q_rows * 128));
                for (int p = 0; p < L::NP; ++p)
                    tma_load_2d(smem + L::OFF_Q + p * L::PANEL_Q, mq, p * 64, q_row0, &x.q_full);
            }
            int armed = 0;  // tiles whose loads were issued
            for (int i = 0; i < n_tiles; ++i) {
                const int nb = min(2, cnt - 2 * i);
                int rows[2] = {0, 0}, first[2] = {0, 0};
                for (int h = 0; h < nb; ++h) {
                    const int g = __ldg(lst + 2 * i + h);
                    rows[h] = block_rows(a, g, bh, &first[h]);
                    if (rows[h] == 0 && is_k) record_error(a.err, DEVERR_LIST | 2);
                }
                const uint32_t bytes = static_cast<uint32_t>((rows[0] + rows[1]) * 128 * L::NP);
                const int s = i % nslots;
                if (!mbar_wait(&empty[s], ((i / nslots) & 1) ^ 1, abort_flag, a.err, is_k ? 0x10 : 0x11)) break;
                if (bytes) mbar_arrive_expect_tx(&full[s], bytes);
                else mbar_arrive(&full[s]);
                for (int h = 0; h < nb; ++h)
                    if (rows[h]) load_block<D, IL>(base + s * slot_bytes, h, rows[h], first[h], mfull, mpart, &full[s]);
                armed = i + 1;
            }
            if (*abort_flag) {
                // Let every copy already issued land before the CTA exits.
                if (is_k) mbar_drain(&x.q_full, 0, 10000000ull);
                for (int i = max(0, armed - nslots); i < armed; ++i)
                    mbar_drain(&full[i % nslots], (i / nslots) & 1, 10000000ull);
            }
        }
    } else if (warp == W_MMA) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 64, false, false);
            constexpr uint32_t IDESC_O = idesc_bf16_f32(128, 64, true, true);
            const uint32_t sQ = smem_u32(smem + L::OFF_Q);
            const uint32_t sK = smem_u32(smem + L::OFF_K);
            const uint32_t sV = smem_u32(smem + L::OFF_V);
            const uint32_t sP = smem_u32(smem + L::OFF_P);
            bool issued_any = false;
            bool ok = mbar_wait(&x.q_full, 0, abort_flag, a.err, 0x20);
            int next_s = 0, next_pv = 0;
            unsigned long long stall_t0 = 0;
            uint32_t idle = 0;
            while (ok && next_pv < n_tiles) {
                bool progressed = false;
                // PV for the oldest tile whose P and V are ready (frees a V slot and a P buffer).
                if (next_pv < next_s) {
                    const int i = next_pv, g = i & 1, vs = i % VSLOTS;
                    if (mbar_test(&x.p_full[g], (i >> 1) & 1) && mbar_test(&x.v_full[vs], (i / VSLOTS) & 1)) {
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            // A = V^T (M = head_dim, MN-major: 64-wide panels LBO apart, 8-row K groups SBO apart)
                            const uint64_t ad = sdesc_sw128(sV + vs * L::V_SLOT + kk * L::KV_K16, L::KV_PANEL, L::KV_SBO);
                            // B = P^T (N = 64 queries, MN-major, one 64-wide panel)
                            const uint64_t bd = sdesc_sw128(sP + g * L::P_BUF + kk * 2048, L::P_BUF, 1024);
                            umma_bf16(tmem + 256u + 64u * g, ad, bd, IDESC_O, (i >= 2 || kk > 0) ? 1u : 0u);
                        }
                        umma_commit(&x.v_empty[vs]);
                        umma_commit(&x.p_empty[g]);
                        issued_any = true;
                        ++next_pv;
                        progressed = true;
                    }
                }
                // S for the next tile once its TMEM buffer is free and its K has landed.
                if (next_s < n_tiles) {
                    const int i = next_s, b = i & 3, ks = i % KSLOTS;
                    const bool buf_free = i < 4 || mbar_test(&x.s_free[b], ((i >> 2) - 1) & 1);
                    if (buf_free && mbar_test(&x.k_full[ks], (i / KSLOTS) & 1)) {
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint32_t panel = static_cast<uint32_t>(kk >> 2);
                            // A = K tile (M = 128 KV rows, K-major), B = Q (N = 64 queries, K-major)
                            const uint64_t ad =
                                sdesc_sw128(sK + ks * L::K_SLOT + panel * L::KV_PANEL + (kk & 3) * 32, 16, L::KV_SBO);
                            const uint64_t bd = sdesc_sw128(sQ + panel * L::PANEL_Q + (kk & 3) * 32, 16, 1024);
                            umma_bf16(tmem + 64u * b, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
                        }
                        umma_commit(&x.k_empty[ks]);
                        umma_commit(&x.s_full[b]);
                        issued_any = true;
                        ++next_s;
                        progressed = true;
                    }
                }
                if (progressed) {
                    idle = 0;
                } else if (++idle == 1) {
                    stall_t0 = globaltimer();
                } else if ((idle & 63u) == 0u) {
                    if (*abort_flag) break;
                    if (globaltimer() - stall_t0 > LF_WAIT_LIMIT_NS) {
                        *abort_flag = 1;
                        record_error(a.err, DEVERR_TIMEOUT | 0x22);
                        break;
                    }
                }
            }
            if (*abort_flag && issued_any) {
                umma_commit(&x.drain);
                mbar_drain(&x.drain, 0, 10000000ull);
            }
        }
    } else if (warp >= W_SOFT0) {
        // ------------------------------------------------------------ softmax
        const int g = (warp - W_SOFT0) >> 2;   // this warpgroup takes the tiles i with i % 2 == g
        const int sp = warp & 3;               // TMEM sub-partition of this warp
        const int t = sp * 32 + lane;          // KV token of a tile / head-dim row of O^T
        const int bar_id = 1 + g;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(sp * 32) << 16);
        const uint32_t o_col = 256u + 64u * static_cast<uint32_t>(g);
        const float sl2 = a.scale_log2;
        uint8_t* pbuf = smem + L::OFF_P + g * L::P_BUF + (t >> 3) * 1024 + (t & 7) * 128;
        float l[64];  // this thread's share of each column's softmax denominator
#pragma unroll
        for (int c = 0; c < 64; ++c) l[c] = 0.f;

        for (int i = g; i < n_tiles; i += 2) {
            const int j = i >> 1;  // local tile index of this warpgroup
            const int bi = 2 * i + (t >> 6);
            int rows = 0;
            if (bi < cnt) {
                if (bi < ROWS_SMEM) {
                    rows = x.rows[bi];
                } else {
                    int first;
                    rows = block_rows(a, __ldg(lst + bi), bh, &first);
                }
            }
            const bool valid = (t & 63) < rows;
            const uint32_t s_addr = lane_base + 64u * static_cast<uint32_t>(i & 3);
            mbar_wait(&x.s_full[i & 3], (i >> 2) & 1, abort_flag, a.err, 0x30);
            __syncwarp();
            tc_fence_after();
            // 1. Does any score exceed the stabiliser by more than the lazy bound?
            float xmax = -INFINITY;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float s[32];
                tmem_ld32(s_addr + 32u * h, s);
                tmem_ld_wait();
#pragma unroll
                for (int c = 0; c < 32; c += 4) {
                    const float4 m4 = *reinterpret_cast<const float4*>(&x.m_s[g][32 * h + c]);
                    s[c] = fmaf(s[c], sl2, -m4.x);
                    s[c + 1] = fmaf(s[c + 1], sl2, -m4.y);
                    s[c + 2] = fmaf(s[c + 2], sl2, -m4.z);
                    s[c + 3] = fmaf(s[c + 3], sl2, -m4.w);
                }
#pragma unroll
                for (int w = 16; w >= 1; w >>= 1)
#pragma unroll
                    for (int c = 0; c < w; ++c) s[c] = fmaxf(s[c], s[c + w]);
                xmax = fmaxf(xmax, s[0]);
            }
            if (!valid) xmax = -INFINITY;
            const bool need = named_bar_or(bar_id, 128, xmax > LAZY_RESCALE_LOG2);
            // PV of this warpgroup's previous tile must be done before its P
            // buffer is rewritten or its O^T columns are rescaled.
            if (j > 0) mbar_wait(&x.p_empty[g], (j - 1) & 1, abort_flag, a.err, 0x31);
            __syncwarp();
            if (need) {
                // 2. Exact column maxima of this tile over its 128 KV tokens.
                __syncwarp();
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float s[32];
                    tmem_ld32(s_addr + 32u * h, s);
                    tmem_ld_wait();
#pragma unroll
                    for (int c = 0; c < 32; ++c) s[c] = valid ? s[c] * sl2 : -INFINITY;
                    transpose_reduce<true>(s, lane);
                    x.red[g][sp][32 * h + lane] = s[0];
                }
                named_bar_sync(bar_id, 128);
                float alpha[2], m_new[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int c = 32 * h + lane;  // lane owns column c of this half
                    const float m_old = x.m_s[g][c];
                    m_new[h] = fmaxf(m_old, fmaxf(fmaxf(x.red[g][0][c], x.red[g][1][c]),
                                                  fmaxf(x.red[g][2][c], x.red[g][3][c])));
                    alpha[h] = (m_new[h] == -INFINITY) ? 1.f : fast_exp2(m_old - m_new[h]);
                }
                named_bar_sync(bar_id, 128);  // every warp has read the old maxima
                if (sp == 0) {
                    x.m_s[g][lane] = m_new[0];
                    x.m_s[g][32 + lane] = m_new[1];
                }
                tc_fence_after();
                __syncwarp();
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if (j > 0) {
                        float o[32];
                        tmem_ld32(lane_base + o_col + 32u * h, o);
                        tmem_ld_wait();
#pragma unroll
                        for (int c = 0; c < 32; ++c) o[c] *= __shfl_sync(0xffffffffu, alpha[h], c);
                        tmem_st32(lane_base + o_col + 32u * h, o);
                    }
#pragma unroll
                    for (int c = 0; c < 32; ++c) l[32 * h + c] *= __shfl_sync(0xffffffffu, alpha[h], c);
                }
                if (j > 0) tmem_st_wait();
                named_bar_sync(bar_id, 128);
            }
            // 3. Probabilities P = 2^(s*scale*log2e - m) as bf16 P^T rows.
            __syncwarp();
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                float s[32];
                tmem_ld32(s_addr + 32u * h, s);
                tmem_ld_wait();
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 32; c += 4) {
                    const float4 m4 = *reinterpret_cast<const float4*>(&x.m_s[g][32 * h + c]);
                    const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
                    for (int e = 0; e < 4; e += 2) {
                        const float p0 = valid ? fast_exp2(fmaf(s[c + e], sl2, -mm[e])) : 0.f;
                        const float p1 = valid ? fast_exp2(fmaf(s[c + e + 1], sl2, -mm[e + 1])) : 0.f;
                        l[32 * h + c + e] += p0;
                        l[32 * h + c + e + 1] += p1;
                        pk[(c + e) >> 1] = pack_bf16x2(p0, p1);
                    }
                }
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int chunk = (4 * h + k) ^ (t & 7);
                    *reinterpret_cast<uint4*>(pbuf + chunk * 16) =
                        make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&x.s_free[i & 3]);
                mbar_arrive(&x.p_full[g]);
            }
        }

        // ------------------------------------------------------------ epilogue
        const int n_g = (n_tiles - g + 1) >> 1;  // tiles this warpgroup took
        if (n_g > 0) mbar_wait(&x.p_empty[g], (n_g - 1) & 1, abort_flag, a.err, 0x34);
        __syncwarp();
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float v[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) v[c] = l[32 * h + c];
            transpose_reduce<false>(v, lane);
            x.red[g][sp][32 * h + lane] = v[0];
        }
        named_bar_sync(bar_id, 128);
        if (sp == 0) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int c = 32 * h + lane;
                x.lsum[g][c] = x.red[g][0][c] + x.red[g][1][c] + x.red[g][2][c] + x.red[g][3][c];
            }
        }
        tc_fence_before();
        named_bar_sync(3, 256);  // both warpgroups: sums, maxima and last PVs are final
        tc_fence_after();
        // Warpgroup g merges and writes query columns [32g, 32g + 32).
        const int n0 = (n_tiles + 1) >> 1, n1 = n_tiles >> 1;
        float o0[32], o1[32];
        __syncwarp();
        if (n0 > 0) {
            tmem_ld32(lane_base + 256u + 32u * g, o0);
        }
        if (n1 > 0) {
            tmem_ld32(lane_base + 320u + 32u * g, o1);
        }
        tmem_ld_wait();
        __nv_bfloat16* ostage = reinterpret_cast<__nv_bfloat16*>(smem + L::OFF_K);
        if (t < D) {
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                const int cc = 32 * g + c;
                const float m0 = x.m_s[0][cc], m1 = x.m_s[1][cc];
                const float mx = fmaxf(m0, m1);
                const float f0 = (n0 > 0 && m0 != -INFINITY) ? fast_exp2(m0 - mx) : 0.f;
                const float f1 = (n1 > 0 && m1 != -INFINITY) ? fast_exp2(m1 - mx) : 0.f;
                const float den = x.lsum[0][cc] * f0 + x.lsum[1][cc] * f1;
                const float num = (f0 != 0.f ? o0[c] * f0 : 0.f) + (f1 != 0.f ? o1[c] * f1 : 0.f);
                ostage[cc * D + t] = __float2bfloat16_rn(den > 0.f ? num / den : 0.f);
            }
        }
        named_bar_sync(3, 256);
        const int chunks = q_rows * (D / 8);
        for (int idx = tid - W_SOFT0 * 32; idx < chunks; idx += 256) {
            const int qq = idx / (D / 8);
            const int c8 = idx - qq * (D / 8);
            *reinterpret_cast<uint4*>(a.out + (static_cast<long long>(q_row0) + qq) * D + c8 * 8) =
                *reinterpret_cast<const uint4*>(ostage + qq * D + c8 * 8);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == W_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

template <int D, bool IL>
cudaError_t launch_attn_t(const AttnMaps& m, const AttnArgs& a, int n_rows, cudaStream_t s)
{
    constexpr uint32_t smem = attn_smem_bytes<D, IL>();
    static_assert(smem <= 232448, "shared memory plan exceeds 227 KB");
    static int configured_device = -1;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (configured_device != dev) {
        e = cudaFuncSetAttribute(attn_kernel<D, IL>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        configured_device = dev;
    }
    attn_kernel<D, IL><<<static_cast<unsigned>(n_rows), ATTN_THREADS, smem, s>>>(m.q, m.q_rem, m.k, m.k_rem, m.v,
                                                                               m.v_rem, a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn(const AttnMaps& m, const AttnArgs& a, int D, bool interleaved, int n_rows, cudaStream_t s)
{
    if (n_rows <= 0) return cudaSuccess;
    if (D == 128)
        return interleaved ? launch_attn_t<128, true>(m, a, n_rows, s) : launch_attn_t<128, false>(m, a, n_rows, s);
    return launch_attn_t<64, false>(m, a, n_rows, s);
}

}  // namespace lf
