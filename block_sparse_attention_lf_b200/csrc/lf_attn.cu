// lf_attn.cu -- block-sparse softmax attention of one HSA call on sm_100a
// tensor cores ("Light Forcing：通过稀疏注意力加速自回归视频扩散",
// paper.rainbus.top, execution flow, stage 3, final step: attention computed
// only over the kept (frame, block) pairs of B_r).
//
// Design (B200-first; the pages' kernel is prior art only):
//   * One CTA per query block (64 query tokens of one head, its own KV block
//     list). CTAs are ordered head-major so a head's K/V stay L2-resident while
//     its query blocks run.
//   * A tile is two listed KV blocks (128 tokens); a step is two tiles. The
//     scores of a step are two M = 64 MMAs, S_h = Q * K_tile(h)^T (M = 64
//     queries, N = 128 keys, K = head_dim), written to the two halves of the
//     TMEM lanes: query row r of tile h lands in lane 32*(r/16) + 16*h + r%16.
//     A softmax thread therefore owns one query row of one tile, so row maxima
//     and row sums need no cross-thread reduction (the two threads of a row,
//     lanes l and l^16, exchange one value per step).
//   * P goes to shared memory as bf16 in the 128-byte-swizzled K-major layout
//     of the PV MMA's B operand, and O^T += V_block^T * P^T runs KV-major
//     (M = 128 head-dim rows, N = 64 queries, K = 16 keys per instruction),
//     which keeps that MMA at M = 128 (M = 64 issues at half rate).
//   * Gather. For head_dim 128 each 64-token block (16 KB, contiguous) arrives
//     as ONE 4-D TMA box {64 elems, 8 rows, 2 panels, 8 row groups} that lands
//     in an interleaved layout [row group][panel][8 rows x 128 B] (128-byte
//     swizzle) with a uniform 2 KB row-group stride, so one descriptor spans a
//     tile's two blocks (K, SBO = 2 KB, panel at +1 KB) and a V block is read
//     MN-major (LBO = 1 KB between head-dim panels, SBO = 2 KB between 8-row
//     groups). Frames whose token count is not a multiple of 8, and head_dim
//     64, use 2-D boxes per 64-wide panel into a plain [panel][row] layout.
//     The K ring holds two tiles but is filled and released per block: each block's
//     score MMAs (M = 64, N = 64, the same rate as N = 128) release its slot, so the next
//     step's first block loads while the tile's second block is still being scored
//     (1-2 % faster than releasing whole tiles). V arrives per block (ring of 4 blocks).
//   * Warp roles (384 threads): warp 0 issues the Q and K loads, warp 1 the V
//     loads, warp 2 allocates TMEM and issues the score MMAs, warp 3 issues the
//     PV MMAs, warps 4-11 are two softmax warpgroups. Warpgroup g takes
//     the steps s with s % 2 == g, with its own running maxima and its own O^T
//     accumulator in TMEM; the two partial softmaxes are merged once in the
//     epilogue (O = (O_0 2^(m_0-M) + O_1 2^(m_1-M)) / (l_0 2^(m_0-M) + l_1 2^(m_1-M))).
//   * Online softmax in fp32, base 2, with a lazy stabiliser: each query row
//     keeps m (running max of scale*log2(e)*score); a step whose scores stay
//     within m + 8 (p <= 256) is exponentiated against the current m; only when
//     some row exceeds that bound does the warpgroup move m and rescale the
//     matching O^T columns in TMEM.
//   * Pipelines: three S buffers in TMEM, a P buffer per warpgroup (a warpgroup
//     rewrites its P once the PV of its previous step is done), per-block V
//     release. Two MMA warps, each in step order with blocking waits: one issues
//     the score MMAs (up to three steps ahead, bounded by the S buffers), the
//     other the PV MMAs; their commits track only their own MMAs and no
//     ordering between the two streams is needed (the S and O^T regions are
//     disjoint, a warpgroup only waits for its own PVs). A lone issuing warp has
//     no other warp to hide its instruction latencies, so each warp's per-step
//     code path (waits, descriptors from precomputed bases, commits) is kept
//     short: a single polling scheduler that tested every barrier each round
//     left the tensor pipe idle more than half of the time.
//   * Every mbarrier wait is bounded (1 s); on expiry the CTA sets an abort
//     flag and the device error word, every role runs its remaining steps
//     without waiting, in-flight copies and MMAs are drained, TMEM is freed,
//     and the kernel returns.
//   * Split of the last wave (optional, AttnArgs::pieces > 0): query blocks
//     past n_whole would run as a last, partial wave on a few SMs, so each of
//     their lists is cut into `pieces` consecutive pieces, one CTA each. Such
//     a CTA runs the same code on its sub-list and ends by writing normalised
//     fp32 rows and each row's (max, denominator) instead of bf16 output;
//     attn_merge_kernel then combines the pieces of each row the way the
//     online softmax would.
#include "lf_device.cuh"
#include "lf_internal.h"

#include <cuda_bf16.h>

#include <cstddef>

namespace lf {
namespace {

constexpr int ATTN_THREADS = 384;
constexpr int W_KPROD = 0, W_VPROD = 1, W_MMA = 2, W_PV = 3, W_SOFT0 = 4;
// K ring (tiles of two blocks) and V ring (single blocks). e4m3 K tiles take half the
// bytes of bf16 ones: the e4m3 kernel holds four K tiles (eight blocks, 64 KB) and four V
// blocks, 2-4 % faster than two K tiles with six V blocks or three with five.
template <bool F8> struct Rings { static constexpr int K = 2, V = 4; };
template <> struct Rings<true> { static constexpr int K = 4, V = 4; };
constexpr int SBUFS = 3;    // S buffers in TMEM (one per step in flight)
constexpr float LAZY_RESCALE_LOG2 = 8.0f;  // p may reach 2^8 before the stabiliser moves
constexpr uint32_t TMEM_COLS = 512;         // S buffer b: columns 128*b; O^T of warpgroup g: 384 + 64*g
constexpr uint32_t TM_O = 384;
constexpr int LIST_SMEM = 1024;             // list entries staged in shared memory

// Shared-memory plan. IL selects the interleaved K/V layout (head_dim 128,
// one 4-D box per block); otherwise K/V use [panel][rows x 128 B].
template <int D, bool IL, bool F8 = false>
struct AttnLayout {
    static constexpr int KSLOTS = Rings<F8>::K;
    static constexpr int VSLOTS = Rings<F8>::V;
    static constexpr int NP = D / 64;                    // 64-element panels of head_dim (bf16)
    static constexpr int NPQ = F8 ? 1 : NP;               // 128-byte panels of a Q / K row
    static constexpr uint32_t PANEL_Q = 64u * 128u;       // 64 rows x 128 B
    static constexpr uint32_t BLOCK_IL = 16384u;          // one 64 x 128 bf16 block (interleaved)
    static constexpr uint32_t Q_BYTES = NPQ * PANEL_Q;
    static constexpr uint32_t K_SLOT = NPQ * 128u * 128u; // a tile: 128 rows
    static constexpr uint32_t V_SLOT = 2u * 64u * 128u;   // a block; the PV MMA has M = 128 head-dim rows
    static constexpr uint32_t P_PANEL = 64u * 128u;       // 64 queries x 64 keys bf16
    static constexpr uint32_t P_BYTES = 4u * P_PANEL;     // a step: 256 keys
    static constexpr uint32_t OFF_Q = 0;
    static constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
    static constexpr uint32_t OFF_V = OFF_K + KSLOTS * K_SLOT;
    static constexpr uint32_t OFF_P = OFF_V + VSLOTS * V_SLOT;
    static constexpr uint32_t OFF_SK = OFF_P + 2 * P_BYTES;  // e4m3: a step's key scales, per warpgroup, two steps
    static constexpr uint32_t OFF_AUX = OFF_SK + (F8 ? 2u * 2u * 256u * 4u : 0u);
    // K tile (B operand of the S MMA, K-major): 8-row group stride and panel offset
    static constexpr uint32_t K_SBO = (IL && !F8) ? 2048u : 1024u;
    static constexpr uint32_t K_PANEL = IL ? 1024u : 128u * 128u;
    // V block (A operand of the PV MMA, MN-major): head-dim panel stride (LBO),
    // 8-row group stride (SBO), and the step between 16-key k-slices
    static constexpr uint32_t V_LBO = IL ? 1024u : 64u * 128u;
    static constexpr uint32_t V_SBO = IL ? 2048u : 1024u;
    static constexpr uint32_t V_K16 = IL ? 4096u : 2048u;
    static_assert(!IL || D == 128, "interleaved layout is for head_dim 128");
    static_assert(!F8 || D == 128, "the e4m3 path is for head_dim 128");
};

template <bool F8>
struct AttnAux {
    static constexpr int KSLOTS = Rings<F8>::K;
    static constexpr int VSLOTS = Rings<F8>::V;
    uint64_t q_full;
    uint64_t k_full[2 * KSLOTS], k_empty[2 * KSLOTS];  // per KV block of the K ring
    uint64_t v_full[VSLOTS], v_empty[VSLOTS];
    uint64_t s_full[SBUFS], s_free[SBUFS];
    uint64_t p_full[2], p_empty[2];  // per warpgroup: its P written / its last PV done
    uint64_t drain, drain_pv;
    uint32_t tmem_base;
    int abort;
    alignas(16) float alpha[2][64];  // per-warpgroup rescale factors of the query columns
    float lsum[2][64];               // softmax denominators of each warpgroup's rows
    alignas(16) float m_s[2][64];    // final running max (log2 units) per warpgroup and query row
    float wgt[2][64];                // epilogue weights of the two accumulators per query row
    int lst[LIST_SMEM];              // the CTA's block list (entries past LIST_SMEM stay in global memory)
};

static_assert(offsetof(AttnAux<false>, alpha) % 16 == 0, "alpha is read with 16-byte loads");
static_assert(offsetof(AttnAux<true>, alpha) % 16 == 0, "alpha is read with 16-byte loads");

template <int D, bool IL, bool F8>
constexpr uint32_t attn_smem_bytes()
{
    return AttnLayout<D, IL, F8>::OFF_AUX + static_cast<uint32_t>(sizeof(AttnAux<F8>)) + 1024u;
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

// List entry b, from the shared-memory copy when it holds it.
__device__ __forceinline__ int list_entry(const int* lst_s, const int* lst, int b)
{
    return b < LIST_SMEM ? lst_s[b] : __ldg(lst + b);
}

// Valid rows of list entry b (0 past the end of the list or for a bad id).
__device__ __forceinline__ int entry_rows(const AttnArgs& a, const int* lst_s, const int* lst, int b, int cnt)
{
    if (b >= cnt) return 0;
    const int g = list_entry(lst_s, lst, b);
    if (g < 0 || g >= a.Nkv) return 0;
    return (g % a.bpf == a.bpf - 1) ? a.rem : 64;
}

// Load one KV block (`rows` valid tokens starting at flattened row `first`)
// to `dst`; `panel_stride` separates the 64-wide panels of the plain layout.
// Called by a converged producer warp; one elected lane issues the copies.
template <int D, bool IL>
__device__ __forceinline__ void load_block(uint8_t* dst, uint32_t panel_stride, int rows, int first,
                                           const CUtensorMap* full, const CUtensorMap* part, uint64_t* bar)
{
    using L = AttnLayout<D, IL>;
    const CUtensorMap* m = rows == 64 ? full : part;
    if constexpr (IL) {
        tma_load_4d_elect(dst, m, 0, 0, 0, first >> 3, bar);
    } else {
#pragma unroll
        for (int p = 0; p < L::NP; ++p) tma_load_2d_elect(dst + p * panel_stride, m, p * 64, first, bar);
    }
}

// 128 consecutive fp32 columns of this thread's TMEM lane (issued as four
// loads; the caller waits).
__device__ __forceinline__ void tmem_ld128_nowait(uint32_t taddr, float (&v)[128])
{
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint32_t r[32];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
            "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
            "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
              "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
              "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
              "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
              "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
              "=r"(r[31])
            : "r"(taddr + 32u * q));
#pragma unroll
        for (int i = 0; i < 32; ++i) v[32 * q + i] = __uint_as_float(r[i]);
    }
}

template <int D, bool IL, bool F8>
__global__ void __launch_bounds__(ATTN_THREADS, 1)
attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_q_rem,
            const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_k_rem,
            const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_v_rem,
            const AttnArgs a)
{
    using L = AttnLayout<D, IL, F8>;
    constexpr int KSLOTS = L::KSLOTS, VSLOTS = L::VSLOTS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    AttnAux<F8>& x = *reinterpret_cast<AttnAux<F8>*>(smem + L::OFF_AUX);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // the merge kernel of a split call may be scheduled once every CTA has started
    // (it waits for this grid's completion before reading anything)
    if (tid == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // launched as a programmatic dependent of the selection: its lists (and any earlier
    // kernel's q, k, v) are complete and visible once this returns
    asm volatile("griddepcontrol.wait;" ::: "memory");
    int row = blockIdx.x;
    int slot = -1;  // partial-result slot of a CTA that computes one piece of a list
    if (a.pieces > 0 && row >= a.n_whole) {
        slot = row - a.n_whole;
        row = a.n_whole + slot / a.pieces;
    }
    const int bh = row / a.Rq;
    const int r = row - bh * a.Rq;
    int cnt = __ldg(a.block_count + row);
    if (cnt < 0 || cnt > a.list_cap) {
        if (tid == 0) record_error(a.err, DEVERR_LIST | 1);
        cnt = cnt < 0 ? 0 : a.list_cap;
    }
    const int* lst = a.block_list + static_cast<long long>(row) * a.list_cap;
    if (slot >= 0) {
        // entries [piece * cnt / pieces, (piece + 1) * cnt / pieces) of the list
        const int piece = slot % a.pieces;
        const int lo = static_cast<int>(static_cast<long long>(piece) * cnt / a.pieces);
        const int hi = static_cast<int>(static_cast<long long>(piece + 1) * cnt / a.pieces);
        lst += lo;
        cnt = hi - lo;
    }
    const int n_tiles = (cnt + 1) >> 1;
    const int n_steps = (n_tiles + 1) >> 1;
    const int fq = r / a.bpf;
    const int jq = r - fq * a.bpf;
    const int q_rows = (jq == a.bpf - 1) ? a.rem : 64;
    const int q_row0 = bh * a.Lq + fq * a.F + jq * 64;

    if (tid == 0) {
        mbar_init(&x.q_full, 1);
        for (int s = 0; s < 2 * KSLOTS; ++s) { mbar_init(&x.k_full[s], 1); mbar_init(&x.k_empty[s], 1); }
        for (int s = 0; s < VSLOTS; ++s) { mbar_init(&x.v_full[s], 1); mbar_init(&x.v_empty[s], 1); }
        for (int s = 0; s < SBUFS; ++s) {
            mbar_init(&x.s_full[s], 1);
            mbar_init(&x.s_free[s], 4);  // one arrival per warp of the owning warpgroup
        }
        mbar_init(&x.p_full[0], 4);
        mbar_init(&x.p_full[1], 4);
        mbar_init(&x.p_empty[0], 1);
        mbar_init(&x.p_empty[1], 1);
        mbar_init(&x.drain, 1);
        mbar_init(&x.drain_pv, 1);
        x.abort = 0;
        fence_mbar_init();
    }
    if (warp == W_MMA) {
        tmem_alloc(&x.tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    // The producers and the softmax read the list once per block; keep it on chip.
    for (int b = tid; b < min(cnt, LIST_SMEM); b += ATTN_THREADS) x.lst[b] = __ldg(lst + b);
    // V slots are read in full by the PV MMA (M = 128 head-dim rows); the
    // second panel of a head_dim-64 slot is never loaded and must stay zero,
    // and rows past a partial block must be finite (P is zero there). Q rows
    // past a partial query block only feed discarded output columns.
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

    if (warp == W_KPROD) {
        // ------------------------------------------------------------ K (+ Q) producer (whole warp)
        {
            if (lane == 0) tma_prefetch_desc(&tm_k);
            __syncwarp();
            const CUtensorMap* mq = (q_rows == 64) ? &tm_q : &tm_q_rem;
            mbar_arrive_expect_tx_elect(&x.q_full, static_cast<uint32_t>(L::NPQ * q_rows * 128));
            for (int p = 0; p < L::NPQ; ++p)
                tma_load_2d_elect(smem + L::OFF_Q + p * L::PANEL_Q, mq, p * 64, q_row0, &x.q_full);
            int armed = 0;
            constexpr int KB = 2 * KSLOTS;  // block slots
            for (int e = 0; e < cnt; ++e) {
                int first = 0;
                const int rows = block_rows(a, list_entry(x.lst, lst, e), bh, &first);
                if (rows == 0 && lane == 0) record_error(a.err, DEVERR_LIST | 2);
                const int bi = e % KB;
                if (!mbar_wait(&x.k_empty[bi], ((e / KB) & 1) ^ 1, abort_flag, a.err, 0x10)) break;
                if (rows) mbar_arrive_expect_tx_elect(&x.k_full[bi], static_cast<uint32_t>(rows * 128 * L::NPQ));
                else mbar_arrive_elect(&x.k_full[bi]);
                uint8_t* slot = smem + L::OFF_K + ((e >> 1) % KSLOTS) * L::K_SLOT;
                const int h = e & 1;
                if (rows) {
                    if constexpr (F8) {
                        tma_load_2d_elect(slot + h * 8192u, rows == 64 ? &tm_k : &tm_k_rem, 0, first, &x.k_full[bi]);
                    } else {
                        load_block<D, IL>(slot + h * (IL ? L::BLOCK_IL : 64u * 128u), 128u * 128u, rows, first, &tm_k,
                                          &tm_k_rem, &x.k_full[bi]);
                    }
                }
                armed = e + 1;
            }
            if (*abort_flag) {
                // Let every copy already issued land before the CTA exits.
                mbar_drain(&x.q_full, 0, 10000000ull);
                for (int e = max(0, armed - KB); e < armed; ++e)
                    mbar_drain(&x.k_full[e % KB], (e / KB) & 1, 10000000ull);
            }
        }
    } else if (warp == W_VPROD) {
        // ------------------------------------------------------------ V producer (whole warp)
        {
            if (lane == 0) tma_prefetch_desc(&tm_v);
            __syncwarp();
            int armed = 0;
            for (int b = 0; b < cnt; ++b) {
                int first = 0;
                const int rows = block_rows(a, list_entry(x.lst, lst, b), bh, &first);
                const int s = b % VSLOTS;
                if (!mbar_wait(&x.v_empty[s], ((b / VSLOTS) & 1) ^ 1, abort_flag, a.err, 0x11)) break;
                if (rows) {
                    mbar_arrive_expect_tx_elect(&x.v_full[s], static_cast<uint32_t>(rows * 128 * L::NP));
                    load_block<D, IL>(smem + L::OFF_V + s * L::V_SLOT, 64u * 128u, rows, first, &tm_v, &tm_v_rem,
                                      &x.v_full[s]);
                } else {
                    mbar_arrive_elect(&x.v_full[s]);
                }
                armed = b + 1;
            }
            if (*abort_flag)
                for (int b = max(0, armed - VSLOTS); b < armed; ++b)
                    mbar_drain(&x.v_full[b % VSLOTS], (b / VSLOTS) & 1, 10000000ull);
        }
    } else if (warp == W_MMA || warp == W_PV) {
        // ------------------------------------------------------------ MMA issuers (whole warps,
        // one elected lane issues): warp W_MMA issues the score MMAs of every step in order,
        // warp W_PV the PV MMAs; the waits below are normally already satisfied, which keeps
        // each issuing warp's code path short.
        {
            constexpr uint32_t IDESC_S64 = F8 ? idesc_e4m3_f32(64, 64) : idesc_bf16_f32(64, 64, false, false);
            constexpr uint32_t IDESC_O = idesc_bf16_f32(128, 64, true, false);
            // A descriptor's start field is the byte address >> 4, so an operand at a byte
            // offset o from a base is the base descriptor + (o >> 4).
            const uint64_t dQ = sdesc_sw128(smem_u32(smem + L::OFF_Q), 16, 1024);
            const uint64_t dK = sdesc_sw128(smem_u32(smem + L::OFF_K), 16, L::K_SBO);
            const uint64_t dV = sdesc_sw128(smem_u32(smem + L::OFF_V), L::V_LBO, L::V_SBO);
            const uint64_t dP = sdesc_sw128(smem_u32(smem + L::OFF_P), 16, 1024);
            bool issued_any = false;
            bool ok = mbar_wait(&x.q_full, 0, abort_flag, a.err, 0x20);
            // S of step st: A = Q (M = 64 queries, K-major), B = K tile (N = 128 keys, K-major),
            // tile h of the step into TMEM lanes 16h.. of buffer st % SBUFS.
            auto issue_s = [&](int st) -> bool {
                const int bsel = st % SBUFS;
                if (st >= SBUFS) {
                    if (!mbar_wait(&x.s_free[bsel], ((st / SBUFS) - 1) & 1, abort_flag, a.err, 0x21)) return false;
                    tc_fence_after();  // the softmax's TMEM reads of this buffer come first
                }
                for (int e = 4 * st; e < 4 * st + 4 && e < cnt; ++e) {
                    constexpr int KB = 2 * KSLOTS;
                    const int h = (e >> 1) & 1, b = e & 1;  // tile of the step, block of the tile
                    const int bi = e % KB;
                    if (!mbar_wait(&x.k_full[bi], (e / KB) & 1, abort_flag, a.err, 0x22)) return false;
                    const uint32_t d_addr = tmem + 128u * static_cast<uint32_t>(bsel) + (h ? (16u << 16) : 0u) + 64u * b;
                    const uint32_t boff = F8 ? 8192u : (IL ? L::BLOCK_IL : 64u * 128u);
                    const uint64_t kb = dK + ((static_cast<uint32_t>((e >> 1) % KSLOTS) * L::K_SLOT + b * boff) >> 4);
                    if constexpr (F8) {
#pragma unroll
                        for (int kk = 0; kk < D / 32; ++kk)
                            umma_f8_elect(d_addr, dQ + ((kk * 32) >> 4), kb + ((kk * 32) >> 4), IDESC_S64, kk > 0 ? 1u : 0u);
                    } else {
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint32_t oq = ((kk >> 2) * L::PANEL_Q + (kk & 3) * 32) >> 4;
                            const uint32_t ok_ = ((kk >> 2) * L::K_PANEL + (kk & 3) * 32) >> 4;
                            umma_bf16_elect(d_addr, dQ + oq, kb + ok_, IDESC_S64, kk > 0 ? 1u : 0u);
                        }
                    }
                    umma_commit_elect(&x.k_empty[bi]);
                    issued_any = true;
                }
                umma_commit_elect(&x.s_full[bsel]);
                return true;
            };
            // PV of step st: A = V block^T (M = head_dim, MN-major), B = P^T (N = 64 queries,
            // K-major), into O^T of warpgroup st % 2; V slots are released block by block.
            auto issue_pv = [&](int st) -> bool {
                if (!mbar_wait(&x.p_full[st & 1], (st >> 1) & 1, abort_flag, a.err, 0x23)) return false;
                tc_fence_after();  // an O^T rescale by the softmax comes first
                const uint32_t d_addr = tmem + TM_O + 64u * static_cast<uint32_t>(st & 1);
                for (int q = 0; q < 4; ++q) {
                    const int b = 4 * st + q;
                    if (b >= cnt) break;
                    const int vs = b % VSLOTS;
                    if (!mbar_wait(&x.v_full[vs], (b / VSLOTS) & 1, abort_flag, a.err, 0x24)) return false;
                    const uint64_t vb = dV + ((static_cast<uint32_t>(vs) * L::V_SLOT) >> 4);
                    const uint64_t pb = dP + ((static_cast<uint32_t>(st & 1) * L::P_BYTES + static_cast<uint32_t>(q) * L::P_PANEL) >> 4);
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4)
                        umma_bf16_elect(d_addr, vb + ((k4 * L::V_K16) >> 4), pb + ((k4 * 32) >> 4), IDESC_O,
                                        (st >= 2 || q > 0 || k4 > 0) ? 1u : 0u);
                    umma_commit_elect(&x.v_empty[vs]);
                    issued_any = true;
                }
                umma_commit_elect(&x.p_empty[st & 1]);
                return true;
            };
            if (warp == W_MMA) {
                for (int st = 0; ok && st < n_steps; ++st) ok = issue_s(st);
            } else {
                for (int st = 0; ok && st < n_steps; ++st) ok = issue_pv(st);
            }
            if (*abort_flag && issued_any) {
                uint64_t* dr = warp == W_MMA ? &x.drain : &x.drain_pv;
                umma_commit_elect(dr);
                mbar_drain(dr, 0, 10000000ull);
            }
        }
    } else if (warp >= W_SOFT0) {
        // ------------------------------------------------------------ softmax
        const int g = (warp - W_SOFT0) >> 2;   // this warpgroup takes the steps s with s % 2 == g
        const int sp = warp & 3;               // TMEM sub-partition of this warp
        const int qr = sp * 16 + (lane & 15);  // query row of this thread's S lane
        const int hh = lane >> 4;              // which tile of the step
        const int bar_id = 1 + g;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(sp * 32) << 16);
        const uint32_t o_col = TM_O + 64u * static_cast<uint32_t>(g);
        // Scores of the e4m3 path are S8 = <q8, k8>; the real score is S8 * s_q(row) * s_k(key),
        // so the row's multiplier is scale * log2(e) * s_q(row) and each key's s_k comes per step.
        float sl2 = a.scale_log2;
        if constexpr (F8) sl2 = qr < q_rows ? sl2 * __ldg(a.q_scale + q_row0 + qr) : 0.f;
        // this thread's P row: panels 2*hh and 2*hh+1 (keys 128*hh ... 128*hh+127 of the step)
        uint8_t* prow = smem + L::OFF_P + g * L::P_BYTES + (2 * hh) * L::P_PANEL + qr * 128;
        float m_run = -INFINITY;  // stabiliser of this row (identical in lanes l and l^16)
        float l_run = 0.f;        // this thread's share of the row's softmax denominator

        // e4m3: the key scales of this warpgroup's next step, fetched a step ahead (thread i of
        // the warpgroup holds keys i and i + 128 of the step) so their L2 latency overlaps work
        float kv_next[2] = {0.f, 0.f};
        const int wg_i = (warp - W_SOFT0 - 4 * g) * 32 + lane;
        auto fetch_scales = [&](int st) {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int key = wg_i + 128 * half;
                const int e = 2 * (2 * st + half) + ((key & 127) >> 6);
                const int ri = key & 63;
                float kv = 0.f;
                if (e < cnt) {
                    int first = 0;
                    if (block_rows(a, list_entry(x.lst, lst, e), bh, &first) > ri) kv = __ldg(a.k_scale + first + ri);
                }
                kv_next[half] = kv;
            }
        };
        if constexpr (F8) {
            if (g < n_steps) fetch_scales(g);
        }

        int j = 0;  // local step index of this warpgroup
        for (int s = g; s < n_steps; s += 2, ++j) {
            const int tile = 2 * s + hh;
            const int rows0 = entry_rows(a, x.lst, lst, 2 * tile, cnt);
            const int rows1 = entry_rows(a, x.lst, lst, 2 * tile + 1, cnt);
            const int bsel = s % SBUFS;
            float* sk = nullptr;  // e4m3: this step's 256 key scales in shared memory
            if constexpr (F8) {
                // this step's scales (fetched a step ago) through shared memory to every thread
                sk = reinterpret_cast<float*>(smem + L::OFF_SK) + (g * 2 + (j & 1)) * 256;
                sk[wg_i] = kv_next[0];
                sk[wg_i + 128] = kv_next[1];
                named_bar_sync(bar_id, 128);
                if (s + 2 < n_steps) fetch_scales(s + 2);
            }
            mbar_wait(&x.s_full[bsel], (s / SBUFS) & 1, abort_flag, a.err, 0x30);
            __syncwarp();
            tc_fence_after();
            float sv[128];
            tmem_ld128_nowait(lane_base + 128u * bsel, sv);
            tmem_ld_wait();
            if constexpr (F8) {
                const float* skh = sk + 128 * hh;
#pragma unroll
                for (int c = 0; c < 128; c += 4) {
                    const float4 t4 = *reinterpret_cast<const float4*>(skh + c);
                    fmul2(sv[c], sv[c + 1], t4.x, t4.y);
                    fmul2(sv[c + 2], sv[c + 3], t4.z, t4.w);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&x.s_free[bsel]);
            // 1. Row maximum over the valid keys of the step (masked keys -> -inf).
            if (!__all_sync(0xffffffffu, rows0 == 64 && rows1 == 64)) {
#pragma unroll
                for (int c = 0; c < 128; ++c) {
                    const bool ok = c < 64 ? (c < rows0) : (c - 64 < rows1);
                    sv[c] = ok ? sv[c] : -INFINITY;
                }
            }
            float mx;
            {
                float m3[43];
#pragma unroll
                for (int i = 0; i < 42; ++i) m3[i] = fmax3(sv[3 * i], sv[3 * i + 1], sv[3 * i + 2]);
                m3[42] = fmaxf(sv[126], sv[127]);
                float m2[15];
#pragma unroll
                for (int i = 0; i < 14; ++i) m2[i] = fmax3(m3[3 * i], m3[3 * i + 1], m3[3 * i + 2]);
                m2[14] = m3[42];
                float m1[5];
#pragma unroll
                for (int i = 0; i < 5; ++i) m1[i] = fmax3(m2[3 * i], m2[3 * i + 1], m2[3 * i + 2]);
                mx = fmaxf(fmax3(m1[0], m1[1], m1[2]), fmaxf(m1[3], m1[4]));
            }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const float ms = mx * sl2;
            const bool need = ms > m_run + LAZY_RESCALE_LOG2;
            const float m_new = need ? ms : m_run;
            const float alpha = need ? fast_exp2(m_run - m_new) : 1.f;  // 0 when m_run = -inf
            l_run *= alpha;
            m_run = m_new;
            // 2. Probabilities (registers), then wait until the PV of this warpgroup's
            // previous step has read its P buffer and finished accumulating into its O^T.
            const float mu = (m_run == -INFINITY) ? 0.f : m_run;
            uint32_t pk[64];
            float la = 0.f, lb = 0.f;
#pragma unroll
            for (int c = 0; c < 128; c += 2) {
                float e0, e1;
                ffma2_bc(e0, e1, sv[c], sv[c + 1], sl2, -mu);
                const float p0 = fast_exp2(e0);
                const float p1 = fast_exp2(e1);
                fadd2_acc(la, lb, p0, p1);
                pk[c >> 1] = pack_bf16x2(p0, p1);
            }
            l_run += la + lb;
            if (j > 0) mbar_wait(&x.p_empty[g], (j - 1) & 1, abort_flag, a.err, 0x31);
            // 3. P row -> shared memory (two 64-key panels, 128-byte swizzle).
#pragma unroll
            for (int pp = 0; pp < 2; ++pp) {
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const int chunk = c ^ (qr & 7);
                    const int k = 32 * pp + 4 * c;
                    *reinterpret_cast<uint4*>(prow + pp * L::P_PANEL + chunk * 16) =
                        make_uint4(pk[k], pk[k + 1], pk[k + 2], pk[k + 3]);
                }
            }
            // 4. Rescale O^T columns of rows whose stabiliser moved (rare after the
            // first steps); the previous PV into O^T has completed (waited above).
            if (j > 0 && named_bar_or(bar_id, 128, need)) {
                if (hh == 0) x.alpha[g][qr] = alpha;
                named_bar_sync(bar_id, 128);
                tc_fence_after();
                __syncwarp();
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float o[32];
                    tmem_ld32(lane_base + o_col + 32u * h, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int c = 0; c < 32; c += 4) {
                        const float4 a4 = *reinterpret_cast<const float4*>(&x.alpha[g][32 * h + c]);
                        o[c] *= a4.x;
                        o[c + 1] *= a4.y;
                        o[c + 2] *= a4.z;
                        o[c + 3] *= a4.w;
                    }
                    tmem_st32(lane_base + o_col + 32u * h, o);
                }
                tmem_st_wait();
                named_bar_sync(bar_id, 128);  // alpha reads done before it is rewritten
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&x.p_full[g]);
        }

        // ------------------------------------------------------------ epilogue
        const float l_row = l_run + __shfl_xor_sync(0xffffffffu, l_run, 16);
        if (hh == 0) {
            x.lsum[g][qr] = l_row;
            x.m_s[g][qr] = m_run;
        }
        // the last PV of the call ends every PV of both warpgroups
        if (j > 0) mbar_wait(&x.p_empty[g], (j - 1) & 1, abort_flag, a.err, 0x34);
        tc_fence_before();
        named_bar_sync(3, 256);  // both warpgroups: sums, maxima and last PVs are final
        tc_fence_after();
        // Warpgroup g merges and writes query columns [32g, 32g + 32).
        const int n0 = (n_steps + 1) >> 1, n1 = n_steps >> 1;
        float o0[32], o1[32];
        __syncwarp();
        tmem_ld32(lane_base + TM_O + 32u * g, o0);
        tmem_ld32(lane_base + TM_O + 64u + 32u * g, o1);
        __nv_bfloat16* ostage = reinterpret_cast<__nv_bfloat16*>(smem + L::OFF_K);
        const int t = sp * 32 + lane;
        // O = O_0 w_0 + O_1 w_1 with w_i = 2^(m_i - M) / l: one division and two
        // exponentials per query row, by the first warp of the warpgroup
        if (t < 32) {
            const int cc = 32 * g + t;
            const float m0 = x.m_s[0][cc], m1 = x.m_s[1][cc];
            const float mx = fmaxf(m0, m1);
            const float f0 = (n0 > 0 && m0 != -INFINITY) ? fast_exp2(m0 - mx) : 0.f;
            const float f1 = (n1 > 0 && m1 != -INFINITY) ? fast_exp2(m1 - mx) : 0.f;
            const float den = x.lsum[0][cc] * f0 + x.lsum[1][cc] * f1;
            const float inv = den > 0.f ? 1.f / den : 0.f;
            x.wgt[0][cc] = f0 * inv;
            x.wgt[1][cc] = f1 * inv;
            if (slot >= 0) {
                float* ml = a.part_ml + (static_cast<long long>(slot) * 64 + cc) * 2;
                ml[0] = den > 0.f ? mx : -INFINITY;
                ml[1] = den > 0.f ? den : 0.f;
            }
        }
        tmem_ld_wait();
        named_bar_sync(bar_id, 128);  // this warpgroup's weights are visible
        if (slot >= 0) {
            // one piece of a list: normalised fp32 rows for the merge kernel (a warp
            // stores 32 consecutive floats of one row at a time)
            if (t < D) {
                float* po = a.part_o + static_cast<long long>(slot) * 64 * D + t;
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const int cc = 32 * g + c;
                    const float w0 = x.wgt[0][cc], w1 = x.wgt[1][cc];
                    po[static_cast<long long>(cc) * D] = (w0 != 0.f ? o0[c] * w0 : 0.f) + (w1 != 0.f ? o1[c] * w1 : 0.f);
                }
            }
        } else {
            if (t < D) {
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const int cc = 32 * g + c;
                    const float w0 = x.wgt[0][cc], w1 = x.wgt[1][cc];
                    ostage[cc * D + t] = __float2bfloat16_rn((w0 != 0.f ? o0[c] * w0 : 0.f) + (w1 != 0.f ? o1[c] * w1 : 0.f));
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
    }

    tc_fence_before();
    __syncthreads();
    if (warp == W_MMA) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// Merge of the list pieces of the query blocks past n_whole: with (M_p, L_p) the
// max and denominator of piece p and O_p its normalised rows,
//   out = sum_p 2^(M_p - M) L_p O_p / sum_p 2^(M_p - M) L_p,   M = max_p M_p,
// the same softmax over the union of the pieces' keys. A warp per query row,
// eight rows per CTA; lane l holds head-dim elements [V l, V l + V). Lane i
// computes the weight of piece p0 + i, which a shuffle hands to the whole warp,
// so the loads of consecutive pieces are independent.
template <int D>
__global__ void __launch_bounds__(256) attn_merge_kernel(const AttnArgs a)
{
    constexpr int V = D / 32;  // 4 (head_dim 128) or 2 (head_dim 64)
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tr = blockIdx.x >> 3;                     // query block index past n_whole
    const int qq = ((blockIdx.x & 7) << 3) + warp;      // row within the query block
    const int row = a.n_whole + tr;
    const int bh = row / a.Rq;
    const int r = row - bh * a.Rq;
    const int fq = r / a.bpf;
    const int jq = r - fq * a.bpf;
    const int q_rows = (jq == a.bpf - 1) ? a.rem : 64;
    if (qq >= q_rows) return;
    // launched as a programmatic dependent of the attention grid: wait until that
    // grid has finished and its partial rows are visible
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const long long q_row = static_cast<long long>(bh) * a.Lq + fq * a.F + jq * 64 + qq;
    const long long s0 = static_cast<long long>(tr) * a.pieces;
    const float* ml = a.part_ml + (s0 * 64 + qq) * 2;          // piece p at ml[p * 128]
    const float* po = a.part_o + (s0 * 64 + qq) * D + V * lane;  // piece p at po[p * 64 * D]
    float M = -INFINITY;
    for (int p = lane; p < a.pieces; p += 32) M = fmaxf(M, ml[static_cast<long long>(p) * 128]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float acc[V];
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = 0.f;
    float den = 0.f;
    for (int p0 = 0; p0 < a.pieces; p0 += 32) {
        float wl = 0.f;
        if (p0 + lane < a.pieces) {
            const float mp = ml[static_cast<long long>(p0 + lane) * 128];
            if (mp != -INFINITY) wl = fast_exp2(mp - M) * ml[static_cast<long long>(p0 + lane) * 128 + 1];
        }
        den += wl;
        const int np = min(32, a.pieces - p0);
#pragma unroll 4
        for (int i = 0; i < np; ++i) {
            const float w = __shfl_sync(0xffffffffu, wl, i);
            const float* src = po + static_cast<long long>(p0 + i) * 64 * D;
            if constexpr (V == 4) {
                const float4 x = *reinterpret_cast<const float4*>(src);
                acc[0] += w * x.x;
                acc[1] += w * x.y;
                acc[2] += w * x.z;
                acc[3] += w * x.w;
            } else {
                const float2 x = *reinterpret_cast<const float2*>(src);
                acc[0] += w * x.x;
                acc[1] += w * x.y;
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    const float inv = den > 0.f ? 1.f / den : 0.f;
    uint16_t* out = a.out + q_row * D + V * lane;
    if constexpr (V == 4) {
        const uint32_t lo = pack_bf16x2(acc[0] * inv, acc[1] * inv);
        const uint32_t hi = pack_bf16x2(acc[2] * inv, acc[3] * inv);
        *reinterpret_cast<uint2*>(out) = make_uint2(lo, hi);
    } else {
        *reinterpret_cast<uint32_t*>(out) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    }
}

template <int D, bool IL, bool F8>
cudaError_t launch_attn_t(const AttnMaps& m, const AttnArgs& a, cudaStream_t s)
{
    constexpr uint32_t smem = attn_smem_bytes<D, IL, F8>();
    static_assert(smem <= 232448, "shared memory plan exceeds 227 KB");
    static int configured_device = -1;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (configured_device != dev) {
        e = cudaFuncSetAttribute(attn_kernel<D, IL, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        configured_device = dev;
    }
    const int tail = a.pieces > 0 ? a.n_rows - a.n_whole : 0;
    const long long grid = a.n_units;
    {
        // a programmatic dependent launch: the grid may be scheduled while the previous kernel
        // in the stream finishes, and waits for it (griddepcontrol.wait) before reading memory
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(grid));
        cfg.blockDim = dim3(ATTN_THREADS);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, attn_kernel<D, IL, F8>, m.q, m.q_rem, m.k, m.k_rem, m.v, m.v_rem, a);
    }
    if (e != cudaSuccess || tail == 0) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(tail) * 8u);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, attn_merge_kernel<D>, a);
}

}  // namespace

cudaError_t launch_attn(const AttnMaps& m, const AttnArgs& a, int D, bool interleaved, cudaStream_t s)
{
    if (a.n_units <= 0) return cudaSuccess;
    if (D == 128)
        return interleaved ? launch_attn_t<128, true, false>(m, a, s) : launch_attn_t<128, false, false>(m, a, s);
    return launch_attn_t<64, false, false>(m, a, s);
}

cudaError_t launch_attn_fp8(const AttnMaps& m, const AttnArgs& a, bool v_interleaved, cudaStream_t s)
{
    if (a.n_units <= 0) return cudaSuccess;
    return v_interleaved ? launch_attn_t<128, true, true>(m, a, s) : launch_attn_t<128, false, true>(m, a, s);
}

}  // namespace lf
