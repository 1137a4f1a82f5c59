// lf_pool.cu -- token compression of one HSA call ("Light Forcing：通过稀疏注意力
// 加速自回归视频扩散", paper.rainbus.top, execution flow, stage 2: block mean
// pooling of q and k, frame-level compression of the keys; gist.science
// Technical Summary 2.2 "Token Compression").
//
// HBM-bound streaming reduction. A unit is one frame of one (batch, head): the KV
// frames being pooled, then the query frames of the current chunk. Persistent CTAs
// (one per SM) walk units blockIdx.x, +gridDim.x, ...; in each CTA one producer warp
// streams every block of its units (64 tokens x head_dim bf16, 16 KB contiguous at
// head_dim 128) into an 8-slot shared-memory ring with 1-D bulk copies (TMA), so
// 128 KB per SM are in flight whatever the consumers do, and the next unit's blocks
// arrive while the current one finishes. The copies carry an L2 evict-first policy: q and k
// are streamed once here, so their lines are the first replaced and the pooling does not
// evict (and write back) other kernels' lines (30.7 -> 26.7 us at layer480p after a 512 MiB
// write that leaves L2 dirty; 24.6 us either way on a clean L2). Consumer warp w reduces
// blocks w, w+8, ... of each unit from shared memory: lane l sums columns [l*D/32, (l+1)*D/32) over the
// block's rows, so a block's column sums need no shuffle; it writes the block mean
// and keeps a running frame sum. At the end of a K frame the 8 warps' sums are
// combined in warp order (deterministic, and the same for a frame wherever it falls
// in the CTA's sequence) and divided by the frame's token count, so K is read once.
#include "lf_device.cuh"
#include "lf_internal.h"

namespace lf {
namespace {

constexpr int POOL_CONSUMERS = 8;                       // consumer warps
constexpr int POOL_THREADS = 32 * (POOL_CONSUMERS + 1);  // + one producer warp
constexpr int POOL_SLOTS = 8;                            // ring slots of one block each
constexpr int BLOCK_TOKENS = 64;

struct PoolUnit {
    const uint16_t* src;  // first token of the frame
    float* dst;           // its block means
    float* frame;         // its frame mean (K frames), nullptr for query frames
};

__device__ __forceinline__ PoolUnit pool_unit(const PoolArgs& a, int D, long long u)
{
    const int units = a.nk + (a.pool_q ? a.n_cur : 0);
    const int bh = static_cast<int>(u / units);
    const int i = static_cast<int>(u - static_cast<long long>(bh) * units);
    PoolUnit p;
    if (i < a.nk) {
        const int f = a.f0 + i;
        p.src = a.k + (static_cast<long long>(bh) * a.kv_stride + static_cast<long long>(f) * a.F) * D;
        p.dst = a.k_pool + (static_cast<long long>(bh) * a.NF * a.bpf + static_cast<long long>(f) * a.bpf) * D;
        p.frame = a.k_frame + (static_cast<long long>(bh) * a.NF + f) * D;
    } else {
        const int fq = i - a.nk;
        p.src = a.q + (static_cast<long long>(bh) * a.n_cur * a.F + static_cast<long long>(fq) * a.F) * D;
        p.dst = a.q_pool + (static_cast<long long>(bh) * a.n_cur * a.bpf + static_cast<long long>(fq) * a.bpf) * D;
        p.frame = nullptr;
    }
    return p;
}

template <int D>
__global__ void __launch_bounds__(POOL_THREADS, 1) pool_kernel(const PoolArgs a, long long n_units)
{
    constexpr int EPL = D / 32;                                 // columns per lane
    constexpr uint32_t SLOT_BYTES = BLOCK_TOKENS * D * 2;      // one full block
    extern __shared__ __align__(128) uint8_t pool_smem[];
    uint8_t* ring = pool_smem;
    float* red = reinterpret_cast<float*>(pool_smem + POOL_SLOTS * SLOT_BYTES);  // [POOL_CONSUMERS][D]
    uint64_t* full = reinterpret_cast<uint64_t*>(red + POOL_CONSUMERS * D);
    uint64_t* empty = full + POOL_SLOTS;
    int* abort_word = reinterpret_cast<int*>(empty + POOL_SLOTS);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // the selection that follows may be scheduled now; it waits for this grid's completion
    if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (threadIdx.x == 0) {
        for (int s = 0; s < POOL_SLOTS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);  // one consumer warp per block
        }
        *abort_word = 0;
        fence_mbar_init();
    }
    __syncthreads();
    volatile int* abort_flag = abort_word;

    if (warp == POOL_CONSUMERS) {
        // ---------------------------------------------------------------- producer
        long long g = 0;  // blocks issued by this CTA
        const uint64_t pol = l2_policy_evict_first();
        bool ok = true;
        for (long long u = blockIdx.x; ok && u < n_units; u += gridDim.x) {
            const PoolUnit p = pool_unit(a, D, u);
            for (int j = 0; j < a.bpf; ++j, ++g) {
                const int rows = min(BLOCK_TOKENS, a.F - j * BLOCK_TOKENS);
                const int s = static_cast<int>(g % POOL_SLOTS);
                if (!mbar_wait(&empty[s], static_cast<uint32_t>(((g / POOL_SLOTS) & 1) ^ 1), abort_flag, a.err, 0x40)) {
                    ok = false;
                    break;
                }
                const uint32_t bytes = static_cast<uint32_t>(rows) * D * 2;
                mbar_arrive_expect_tx_elect(&full[s], bytes);
                bulk_load_elect_hint(ring + s * SLOT_BYTES, p.src + static_cast<long long>(j) * BLOCK_TOKENS * D, bytes,
                                     &full[s], pol);
            }
        }
        if (!ok)  // let the copies already issued land before the CTA exits
            for (long long g2 = g > POOL_SLOTS ? g - POOL_SLOTS : 0; g2 < g; ++g2)
                mbar_drain(&full[g2 % POOL_SLOTS], static_cast<uint32_t>((g2 / POOL_SLOTS) & 1), 10000000ull);
        return;
    }
    // -------------------------------------------------------------------- consumers
    long long g0 = 0;  // this CTA's blocks before the current unit
    for (long long u = blockIdx.x; u < n_units; u += gridDim.x) {
        const PoolUnit p = pool_unit(a, D, u);
        float facc[EPL];
#pragma unroll
        for (int e = 0; e < EPL; ++e) facc[e] = 0.f;
        for (int j = warp; j < a.bpf; j += POOL_CONSUMERS) {
            const long long g = g0 + j;
            const int s = static_cast<int>(g % POOL_SLOTS);
            const int rows = min(BLOCK_TOKENS, a.F - j * BLOCK_TOKENS);
            // on an expired wait every later wait returns at once: the warps still reach the
            // unit barriers below, so none of them is left waiting there
            if (!mbar_wait(&full[s], static_cast<uint32_t>((g / POOL_SLOTS) & 1), abort_flag, a.err, 0x41)) continue;
            const uint8_t* blk = ring + s * SLOT_BYTES + lane * EPL * 2;
            float acc[EPL];
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
#pragma unroll 8
            for (int r = 0; r < rows; ++r) {
                if constexpr (EPL == 4) {
                    const uint2 w = *reinterpret_cast<const uint2*>(blk + r * D * 2);
                    acc[0] += __uint_as_float(w.x << 16);
                    acc[1] += __uint_as_float(w.x & 0xFFFF0000u);
                    acc[2] += __uint_as_float(w.y << 16);
                    acc[3] += __uint_as_float(w.y & 0xFFFF0000u);
                } else {
                    const uint32_t w = *reinterpret_cast<const uint32_t*>(blk + r * D * 2);
                    acc[0] += __uint_as_float(w << 16);
                    acc[1] += __uint_as_float(w & 0xFFFF0000u);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);  // the slot's bytes are in registers
            const float n = static_cast<float>(rows);
            float* o = p.dst + static_cast<long long>(j) * D + lane * EPL;
            if constexpr (EPL == 4) {
                *reinterpret_cast<float4*>(o) = make_float4(acc[0] / n, acc[1] / n, acc[2] / n, acc[3] / n);
            } else {
                *reinterpret_cast<float2*>(o) = make_float2(acc[0] / n, acc[1] / n);
            }
#pragma unroll
            for (int e = 0; e < EPL; ++e) facc[e] += acc[e];
        }
        g0 += a.bpf;
        // every warp has taken its blocks of this unit before any warp waits on a slot for the
        // next one (a slot's next use must not be waited for before its current use completed)
        named_bar_sync(1, 32 * POOL_CONSUMERS);
        if (p.frame) {
            // frame sum: the consumer warps' partial sums in warp order
#pragma unroll
            for (int e = 0; e < EPL; ++e) red[warp * D + lane * EPL + e] = facc[e];
            named_bar_sync(2, 32 * POOL_CONSUMERS);
            for (int c = threadIdx.x; c < D; c += 32 * POOL_CONSUMERS) {
                float sum = 0.f;
                for (int w = 0; w < POOL_CONSUMERS; ++w) sum += red[w * D + c];
                p.frame[c] = sum / static_cast<float>(a.F);
            }
            named_bar_sync(2, 32 * POOL_CONSUMERS);  // red is read before the next frame rewrites it
        }
    }
}

template <int D>
constexpr size_t pool_smem_bytes()
{
    return static_cast<size_t>(POOL_SLOTS) * BLOCK_TOKENS * D * 2 + POOL_CONSUMERS * D * sizeof(float) +
           2 * POOL_SLOTS * sizeof(uint64_t) + 16;
}

template <int D>
cudaError_t launch_pool_d(const PoolArgs& a, long long n_units, cudaStream_t s)
{
    constexpr size_t smem = pool_smem_bytes<D>();
    static int configured_device = -1;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (configured_device != dev) {
        e = cudaFuncSetAttribute(pool_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        configured_device = dev;
    }
    int sms = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const long long grid = n_units < sms ? n_units : sms;
    pool_kernel<D><<<static_cast<unsigned>(grid), POOL_THREADS, smem, s>>>(a, n_units);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pool(const PoolArgs& a, cudaStream_t s)
{
    const long long n_units = static_cast<long long>(a.BH) * (a.nk + (a.pool_q ? a.n_cur : 0));
    if (n_units <= 0) return cudaSuccess;
    return a.D == 128 ? launch_pool_d<128>(a, n_units, s) : launch_pool_d<64>(a, n_units, s);
}

}  // namespace lf
