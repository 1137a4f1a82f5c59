// lf_api.cu -- the C ABI of liblf_hsa.so (declared in include/lf_hsa.h):
// argument validation, TMA descriptor encoding, kernel launches, the
// Chunk-Aware Growth solver and the per-device error word.
#include "lf_hsa.h"
#include "lf_device.cuh"
#include "lf_internal.h"

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <cudaTypedefs.h>
#include <mutex>

namespace {

__device__ int g_device_error;  // first device-side fault code (0 = none)

constexpr int kMaxDevices = 64;
std::mutex g_mu;

// Device address of the error word on the current device. Looked up on every
// call (a host-side table lookup once the module is loaded), so a context that
// was torn down and re-created never leaves a stale address behind.
lf_status error_word(int** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return LF_ERR_NO_DEVICE;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess || !p) return LF_ERR_CUDA;
    *out = static_cast<int*>(p);
    return LF_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Derived {
    int B, H, D, F, bpf, rem, NF, n_sink, n_recent, n_cur, n_mem, Rq, Nkv, Lq, Lkv;
    long long kv_stride;
};

lf_status check_shape(const lf_hsa_shape* s, Derived* d)
{
    if (!s) return LF_ERR_NULL;
    if (s->batch < 1 || s->heads < 1) return LF_ERR_SHAPE;
    if (s->head_dim != 64 && s->head_dim != 128) return LF_ERR_SHAPE;
    if (s->block_tokens != 64) return LF_ERR_SHAPE;
    if (s->frame_tokens < 1 || s->frame_tokens > 8192) return LF_ERR_SHAPE;
    if (s->n_sink < 0 || s->n_recent < 0 || s->n_cur < 1) return LF_ERR_SHAPE;
    const long long forced = static_cast<long long>(s->n_sink) + s->n_recent + s->n_cur;
    if (s->n_frames < forced) return LF_ERR_SHAPE;
    const long long n_mem = s->n_frames - forced;
    if (n_mem > 1024) return LF_ERR_SHAPE;
    const long long Lkv = static_cast<long long>(s->n_frames) * s->frame_tokens;
    const long long stride = s->kv_stride == 0 ? Lkv : s->kv_stride;
    if (stride < Lkv) return LF_ERR_SHAPE;
    const long long BH = static_cast<long long>(s->batch) * s->heads;
    const long long Lq = static_cast<long long>(s->n_cur) * s->frame_tokens;
    const int bpf = (s->frame_tokens + 63) / 64;
    // TMA coordinates and kernel indices are 32-bit.
    if (BH * stride >= (1ll << 31) || BH * Lq >= (1ll << 31)) return LF_ERR_SHAPE;
    if (BH * s->n_frames * bpf >= (1ll << 31) / 128) return LF_ERR_SHAPE;
    d->B = s->batch;
    d->H = s->heads;
    d->D = s->head_dim;
    d->F = s->frame_tokens;
    d->bpf = bpf;
    d->rem = s->frame_tokens - 64 * (bpf - 1);
    d->NF = s->n_frames;
    d->n_sink = s->n_sink;
    d->n_recent = s->n_recent;
    d->n_cur = s->n_cur;
    d->n_mem = static_cast<int>(n_mem);
    d->Rq = s->n_cur * bpf;
    d->Nkv = s->n_frames * bpf;
    d->Lq = static_cast<int>(Lq);
    d->Lkv = static_cast<int>(Lkv);
    d->kv_stride = stride;
    return LF_OK;
}

int frames_selected(const Derived& d, int chunk_index, int topk_frames)
{
    if (chunk_index == 1) return d.NF;
    const int kf = topk_frames < d.n_mem ? topk_frames : d.n_mem;
    return d.n_sink + kf + d.n_recent + d.n_cur;
}

int blocks_per_frame(const Derived& d, int chunk_index, int topk_blocks)
{
    if (chunk_index == 1) return d.bpf;
    return topk_blocks < d.bpf ? topk_blocks : d.bpf;
}

lf_status launch_status(cudaError_t e) { return e == cudaSuccess ? LF_OK : LF_ERR_CUDA; }

// Bytes of one partial-result slot of the attention split: 64 rows of head_dim
// fp32 values plus a (max, denominator) pair per row.
long long split_slot_bytes(int D) { return 64ll * (D + 2) * 4; }

// Split of the last, partial wave of the one-CTA-per-query-block attention.
// With n_rows query blocks on sm SMs, the last r = n_rows mod sm query blocks
// (all of them when n_rows < sm) would run as a wave of r CTAs on r SMs; their
// lists are cut into k pieces instead. Automatic k (force == 0): sm / r, at most
// list_cap / 8 (a piece of a full list keeps two steps), and no split when sm / r
// is below 8: with the last wave filling more than an eighth of the SMs the
// pieces' own set-up and the merge cost about what the split saves (measured:
// 12 of 148 SMs 344 -> 333 us, 24 of 148 SMs 648 -> 646 and 377 -> 382 us).
// force == 1: no split; force >= 2: k = force. k is capped at list_cap and at
// the slots the workspace holds (slots_cap < 0: unlimited); k < 2: no split.
void split_plan(long long n_rows, int sm, int list_cap, int force, long long slots_cap, int* tail, int* pieces)
{
    *tail = 0;
    *pieces = 0;
    if (n_rows <= 0 || sm <= 0 || force == 1) return;
    const long long r = n_rows % sm;
    if (r == 0) return;
    long long k = force >= 2 ? force : std::min<long long>(sm / r, list_cap / 8);
    if (force == 0 && sm / r < 8) return;
    k = std::min<long long>(k, list_cap);
    if (slots_cap >= 0) k = std::min(k, slots_cap / r);
    if (k < 2) return;
    *tail = static_cast<int>(r);
    *pieces = static_cast<int>(k);
}

lf_status sm_count(int* out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LF_ERR_NO_DEVICE;
    if (cudaDeviceGetAttribute(out, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return LF_ERR_NO_DEVICE;
    return LF_OK;
}

// ---- TMA descriptors ------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D bf16 view [rows, D] with a {64, box_rows} box and 128-byte swizzle.
bool encode_rows(CUtensorMap* m, const void* base, long long rows, int D, int box_rows)
{
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2u};
    const cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1u, 1u};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-D uint8 view [rows, 128] (e4m3 rows of head_dim 128) with a {128, box_rows} box and
// 128-byte swizzle: one box is a block of e4m3 rows.
bool encode_rows_u8(CUtensorMap* m, const void* base, long long rows, int box_rows)
{
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {128u, static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {128u};
    const cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1u, 1u};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 4-D bf16 view of a [rows, 128] tensor as {64 elems, 8 rows, 2 panels,
// rows/8 groups} with a {64, 8, 2, groups} box: one box brings a block of
// 8*groups rows in the interleaved [group][panel][8 rows x 128 B] layout.
bool encode_blocks_il(CUtensorMap* m, const void* base, long long rows, int groups)
{
    auto fn = encode_fn();
    if (!fn || rows % 8 != 0) return false;
    const cuuint64_t dims[4] = {64u, 8u, 2u, static_cast<cuuint64_t>(rows / 8)};
    const cuuint64_t strides[3] = {256u, 128u, 2048u};
    const cuuint32_t box[4] = {64u, 8u, 2u, static_cast<cuuint32_t>(groups)};
    const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

extern "C" {

const char* lf_version(void) { return "lf_hsa 0.1.0 sm_100a"; }

const char* lf_status_string(lf_status s)
{
    switch (s) {
    case LF_OK: return "ok";
    case LF_ERR_NULL: return "a required pointer is NULL";
    case LF_ERR_ALIGN: return "a device pointer is not 16-byte aligned";
    case LF_ERR_SHAPE: return "unsupported shape";
    case LF_ERR_TOPK: return "top-k below 1";
    case LF_ERR_CAP: return "list capacity too small";
    case LF_ERR_INFEASIBLE: return "chunk-aware growth budget is infeasible";
    case LF_ERR_CUDA: return "CUDA error";
    case LF_ERR_DEVICE_TIMEOUT: return "a bounded device wait expired";
    case LF_ERR_ARG: return "invalid argument";
    case LF_ERR_LIST: return "block id or count out of range";
    case LF_ERR_NO_DEVICE: return "no usable CUDA device";
    case LF_ERR_SCRATCH: return "the call needs more than the library's static scratch array";
    }
    return "unknown status";
}

int32_t lf_frames_selected(const lf_hsa_shape* shape, int32_t chunk_index, int32_t topk_frames)
{
    Derived d;
    if (check_shape(shape, &d) != LF_OK || chunk_index < 1 || topk_frames < 1) return -1;
    return frames_selected(d, chunk_index, topk_frames);
}

int32_t lf_list_capacity(const lf_hsa_shape* shape, int32_t chunk_index, int32_t topk_frames, int32_t topk_blocks)
{
    Derived d;
    if (check_shape(shape, &d) != LF_OK || chunk_index < 1 || topk_frames < 1 || topk_blocks < 1) return -1;
    return frames_selected(d, chunk_index, topk_frames) * blocks_per_frame(d, chunk_index, topk_blocks);
}

lf_status lf_pool_range(const lf_hsa_shape* shape, const uint16_t* q, const uint16_t* k, int32_t frame_begin,
                        int32_t frame_end, int32_t pool_q, float* q_pool, float* k_pool, float* k_frame, void* stream)
{
    Derived d;
    lf_status st = check_shape(shape, &d);
    if (st != LF_OK) return st;
    if (frame_begin < 0 || frame_end < frame_begin || frame_end > d.NF) return LF_ERR_ARG;
    if (!k || !k_pool || !k_frame || (pool_q && (!q || !q_pool))) return LF_ERR_NULL;
    if (!aligned16(k) || !aligned16(k_pool) || !aligned16(k_frame) || (pool_q && (!aligned16(q) || !aligned16(q_pool))))
        return LF_ERR_ALIGN;
    int* err = nullptr;
    if ((st = error_word(&err)) != LF_OK) return st;
    lf::PoolArgs a{q, k, q_pool, k_pool, k_frame, d.B * d.H, d.D, d.F, d.bpf, d.NF, d.n_cur, d.kv_stride,
                   frame_begin, frame_end - frame_begin, pool_q ? 1 : 0, err};
    return launch_status(lf::launch_pool(a, static_cast<cudaStream_t>(stream)));
}

lf_status lf_pool(const lf_hsa_shape* shape, const uint16_t* q, const uint16_t* k, float* q_pool, float* k_pool,
                  float* k_frame, void* stream)
{
    if (!q || !q_pool) return LF_ERR_NULL;
    const int32_t nf = shape ? shape->n_frames : 0;
    return lf_pool_range(shape, q, k, 0, nf, 1, q_pool, k_pool, k_frame, stream);
}

lf_status lf_select_frames(const lf_hsa_shape* shape, int32_t chunk_index, int32_t topk_frames, const float* q_pool,
                           const float* k_frame, int32_t* frame_sel, void* stream)
{
    Derived d;
    lf_status st = check_shape(shape, &d);
    if (st != LF_OK) return st;
    if (chunk_index < 1) return LF_ERR_ARG;
    if (topk_frames < 1) return LF_ERR_TOPK;
    if (!q_pool || !k_frame || !frame_sel) return LF_ERR_NULL;
    if (!aligned16(q_pool) || !aligned16(k_frame) || !aligned16(frame_sel)) return LF_ERR_ALIGN;
    lf::SelectFramesArgs a{q_pool, k_frame, frame_sel, d.B * d.H, d.D, d.Rq, d.NF, d.n_sink, d.n_recent,
                           d.n_cur, frames_selected(d, chunk_index, topk_frames), topk_frames, chunk_index};
    return launch_status(lf::launch_select_frames(a, static_cast<cudaStream_t>(stream)));
}

lf_status lf_select_blocks(const lf_hsa_shape* shape, int32_t chunk_index, int32_t topk_frames, int32_t topk_blocks,
                           const float* q_pool, const float* k_pool, const int32_t* frame_sel, int32_t* block_list,
                           int32_t* block_count, int32_t list_cap, void* stream)
{
    Derived d;
    lf_status st = check_shape(shape, &d);
    if (st != LF_OK) return st;
    if (chunk_index < 1) return LF_ERR_ARG;
    if (topk_frames < 1 || topk_blocks < 1) return LF_ERR_TOPK;
    if (!q_pool || !k_pool || !frame_sel || !block_list || !block_count) return LF_ERR_NULL;
    if (!aligned16(q_pool) || !aligned16(k_pool) || !aligned16(frame_sel) || !aligned16(block_list) ||
        !aligned16(block_count))
        return LF_ERR_ALIGN;
    const int n_sel = frames_selected(d, chunk_index, topk_frames);
    const int kb = blocks_per_frame(d, chunk_index, topk_blocks);
    if (list_cap < n_sel * kb) return LF_ERR_CAP;
    int* err = nullptr;
    if ((st = error_word(&err)) != LF_OK) return st;
    lf::SelectBlocksArgs a{q_pool, k_pool, frame_sel, block_list, block_count, d.B * d.H, d.D, d.Rq, d.NF,
                           d.bpf, n_sel, kb, list_cap, chunk_index, err};
    return launch_status(lf::launch_select_blocks(a, static_cast<cudaStream_t>(stream)));
}

lf_status lf_select_mask(const lf_hsa_shape* shape, int32_t chunk_index, int32_t topk_frames, int32_t topk_blocks,
                         const float* q_pool, const float* k_frame, const float* k_pool, int32_t* frame_sel,
                         int32_t* block_list, int32_t* block_count, int32_t list_cap, void* stream)
{
    Derived d;
    lf_status st = check_shape(shape, &d);
    if (st != LF_OK) return st;
    if (chunk_index < 1) return LF_ERR_ARG;
    if (topk_frames < 1 || topk_blocks < 1) return LF_ERR_TOPK;
    if (!q_pool || !k_frame || !k_pool || !frame_sel || !block_list || !block_count) return LF_ERR_NULL;
    if (!aligned16(q_pool) || !aligned16(k_frame) || !aligned16(k_pool) || !aligned16(frame_sel) ||
        !aligned16(block_list) || !aligned16(block_count))
        return LF_ERR_ALIGN;
    const int n_sel = frames_selected(d, chunk_index, topk_frames);
    const int kb = blocks_per_frame(d, chunk_index, topk_blocks);
    if (list_cap < n_sel * kb) return LF_ERR_CAP;
    int* err = nullptr;
    if ((st = error_word(&err)) != LF_OK) return st;
    lf::SelectFramesArgs fa{q_pool, k_frame, frame_sel, d.B * d.H, d.D, d.Rq, d.NF, d.n_sink, d.n_recent,
                            d.n_cur, n_sel, topk_frames, chunk_index};
    lf::SelectBlocksArgs ba{q_pool, k_pool, frame_sel, block_list, block_count, d.B * d.H, d.D, d.Rq, d.NF,
                            d.bpf, n_sel, kb, list_cap, chunk_index, err};
    return launch_status(lf::launch_select_fused(fa, ba, static_cast<cudaStream_t>(stream)));
}

lf_status lf_quant_fp8_rows(const uint16_t* x, int64_t n_rows, int32_t head_dim, uint8_t* x8, float* scales,
                            void* stream)
{
    if (n_rows < 0 || (head_dim != 64 && head_dim != 128)) return LF_ERR_ARG;
    if (n_rows == 0) return LF_OK;
    if (!x || !x8 || !scales) return LF_ERR_NULL;
    if (!aligned16(x) || !aligned16(x8) || !aligned16(scales)) return LF_ERR_ALIGN;
    if (n_rows >= (1ll << 31) * 8) return LF_ERR_SHAPE;
    return launch_status(lf::launch_quant_rows(x, n_rows, head_dim, x8, scales, static_cast<cudaStream_t>(stream)));
}

lf_status lf_select_blocks_1d(const lf_hsa_shape* shape, int32_t chunk_index, int32_t topk_blocks,
                              const float* q_pool, const float* k_pool, int32_t* block_list, int32_t* block_count,
                              int32_t list_cap, void* stream)
{
    Derived d;
    lf_status st = check_shape(shape, &d);
    if (st != LF_OK) return st;
    if (d.Nkv > lf::SEL1D_MAX_NKV) return LF_ERR_SHAPE;
    if (chunk_index < 1) return LF_ERR_ARG;
    if (topk_blocks < 1) return LF_ERR_TOPK;
    if (!q_pool || !k_pool || !block_list || !block_count) return LF_ERR_NULL;
    if (!aligned16(q_pool) || !aligned16(k_pool) || !aligned16(block_list) || !aligned16(block_count))
        return LF_ERR_ALIGN;
    const int keep = (chunk_index == 1 || topk_blocks > d.Nkv) ? d.Nkv : topk_blocks;
    if (list_cap < keep) return LF_ERR_CAP;
    int* err = nullptr;
    if ((st = error_word(&err)) != LF_OK) return st;
    lf::SelectBlocks1dArgs a{q_pool, k_pool, block_list, block_count, d.B * d.H, d.D, d.Rq, d.Nkv,
                             keep, list_cap, chunk_index, err};
    return launch_status(lf::launch_select_blocks_1d(a, static_cast<cudaStream_t>(stream)));
}

lf_status lf_frame_index_build(const lf_hsa_shape* shape, int32_t n_clusters, int32_t iters, const float* k_frame,
                               float* centroids, int32_t* labels, int32_t* offsets, int32_t* members, void* stream)
{
    Derived d;
    lf_status st = check_shape(shape, &d);
    if (st != LF_OK) return st;
    if (n_clusters < 1 || n_clusters > lf::IVF_MAX_CLUSTERS || iters < 0 || iters > 100000) return LF_ERR_ARG;
    if (!k_frame || !centroids || !labels || !offsets || !members) return LF_ERR_NULL;
    if (!aligned16(k_frame) || !aligned16(centroids) || !aligned16(labels) || !aligned16(offsets) ||
        !aligned16(members))
        return LF_ERR_ALIGN;
    const int C = std::min(n_clusters, std::max(d.n_mem, 1));
    lf::FrameIndexArgs a{k_frame, centroids, labels, offsets, members, d.B * d.H, d.D, d.NF, d.n_sink, d.n_mem,
                         C, n_clusters, std::max(d.n_mem, 1), iters};
    return launch_status(lf::launch_frame_index(a, static_cast<cudaStream_t>(stream)));
}

lf_status lf_select_frames_ivf(const lf_hsa_shape* shape, int32_t chunk_index, int32_t topk_frames, int32_t n_clusters,
                               int32_t n_probe, const float* q_pool, const float* k_frame, const float* centroids,
                               const int32_t* offsets, const int32_t* members, int32_t* frame_sel, void* stream)
{
    Derived d;
    lf_status st = check_shape(shape, &d);
    if (st != LF_OK) return st;
    if (chunk_index < 1 || n_clusters < 1 || n_clusters > lf::IVF_MAX_CLUSTERS || n_probe < 1) return LF_ERR_ARG;
    if (topk_frames < 1) return LF_ERR_TOPK;
    if (!q_pool || !k_frame || !centroids || !offsets || !members || !frame_sel) return LF_ERR_NULL;
    if (!aligned16(q_pool) || !aligned16(k_frame) || !aligned16(centroids) || !aligned16(offsets) ||
        !aligned16(members) || !aligned16(frame_sel))
        return LF_ERR_ALIGN;
    const int C = std::min(n_clusters, std::max(d.n_mem, 1));
    lf::SelectFramesIvfArgs a{q_pool, k_frame, centroids, offsets, members, frame_sel, d.B * d.H, d.D, d.Rq, d.NF,
                              d.n_sink, d.n_recent, d.n_cur, d.n_mem, frames_selected(d, chunk_index, topk_frames),
                              topk_frames, chunk_index, C, n_clusters, std::max(d.n_mem, 1), std::min(n_probe, C)};
    return launch_status(lf::launch_select_frames_ivf(a, static_cast<cudaStream_t>(stream)));
}

lf_status lf_attn_split_plan(const lf_hsa_shape* shape, int32_t list_cap, int32_t sm, int32_t* tail_rows,
                             int32_t* pieces, int64_t* workspace_bytes)
{
    Derived d;
    lf_status st = check_shape(shape, &d);
    if (st != LF_OK) return st;
    if (list_cap < 0) return LF_ERR_CAP;
    if (!tail_rows || !pieces || !workspace_bytes) return LF_ERR_NULL;
    if (sm <= 0 && (st = sm_count(&sm)) != LF_OK) return st;
    int t = 0, kp = 0;
    split_plan(static_cast<long long>(d.B) * d.H * d.Rq, sm, list_cap, 0, -1, &t, &kp);
    *tail_rows = t;
    *pieces = kp;
    *workspace_bytes = static_cast<int64_t>(t) * kp * split_slot_bytes(d.D);
    return LF_OK;
}

lf_status lf_block_sparse_attn(const lf_hsa_shape* shape, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                               const int32_t* block_list, const int32_t* block_count, int32_t list_cap,
                               float softmax_scale, uint16_t* out, void* stream)
{
    return lf_block_sparse_attn_ws(shape, q, k, v, block_list, block_count, list_cap, softmax_scale, out, 1, nullptr,
                                   0, stream);
}

lf_status lf_block_sparse_attn_ws(const lf_hsa_shape* shape, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                  const int32_t* block_list, const int32_t* block_count, int32_t list_cap,
                                  float softmax_scale, uint16_t* out, int32_t tail_pieces, void* workspace,
                                  int64_t workspace_bytes, void* stream)
{
    Derived d;
    lf_status st = check_shape(shape, &d);
    if (st != LF_OK) return st;
    if (list_cap < 0) return LF_ERR_CAP;
    if (!(softmax_scale == softmax_scale) || std::isinf(softmax_scale)) return LF_ERR_ARG;
    if (tail_pieces < 0 || workspace_bytes < 0) return LF_ERR_ARG;
    if (!q || !k || !v || !block_list || !block_count || !out) return LF_ERR_NULL;
    if (workspace_bytes > 0 && !workspace) return LF_ERR_NULL;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(block_list) || !aligned16(block_count) ||
        !aligned16(out) || (workspace_bytes > 0 && !aligned16(workspace)))
        return LF_ERR_ALIGN;
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LF_ERR_NO_DEVICE;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return LF_ERR_NO_DEVICE;
    if (major != 10 || minor != 0) return LF_ERR_NO_DEVICE;
    int* err = nullptr;
    if ((st = error_word(&err)) != LF_OK) return st;
    const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(d.D));
    const long long BH = static_cast<long long>(d.B) * d.H;
    lf::AttnMaps m;
    const long long q_rows = BH * d.Lq, kv_rows = BH * d.kv_stride;
    if (!encode_rows(&m.q, q, q_rows, d.D, 64) || !encode_rows(&m.q_rem, q, q_rows, d.D, d.rem)) return LF_ERR_CUDA;
    // One box per KV block when every block starts on an 8-row boundary.
    bool interleaved = d.D == 128 && d.F % 8 == 0 && d.kv_stride % 8 == 0 &&
                       encode_blocks_il(&m.k, k, kv_rows, 8) && encode_blocks_il(&m.k_rem, k, kv_rows, d.rem / 8) &&
                       encode_blocks_il(&m.v, v, kv_rows, 8) && encode_blocks_il(&m.v_rem, v, kv_rows, d.rem / 8);
    if (!interleaved &&
        (!encode_rows(&m.k, k, kv_rows, d.D, 64) || !encode_rows(&m.k_rem, k, kv_rows, d.D, d.rem) ||
         !encode_rows(&m.v, v, kv_rows, d.D, 64) || !encode_rows(&m.v_rem, v, kv_rows, d.D, d.rem)))
        return LF_ERR_CUDA;
    const long long n_rows = BH * d.Rq;
    int tail = 0, pieces = 0;
    if (workspace_bytes > 0 && tail_pieces != 1) {
        int sm = 0;
        if ((st = sm_count(&sm)) != LF_OK) return st;
        split_plan(n_rows, sm, list_cap, tail_pieces, workspace_bytes / split_slot_bytes(d.D), &tail, &pieces);
    }
    float* part_o = static_cast<float*>(workspace);
    float* part_ml = pieces ? part_o + static_cast<long long>(tail) * pieces * 64 * d.D : nullptr;
    lf::AttnArgs a{block_list, block_count, out, list_cap, d.Rq, d.bpf, d.F, d.Lq, d.Nkv, d.rem, d.kv_stride,
                   scale * 1.4426950408889634f, err, static_cast<int>(n_rows - tail), pieces, part_o, part_ml,
                   static_cast<int>(n_rows), static_cast<int>(n_rows - tail + static_cast<long long>(tail) * pieces)};
    return launch_status(lf::launch_attn(m, a, d.D, interleaved, static_cast<cudaStream_t>(stream)));
}

lf_status lf_block_sparse_attn_fp8(const lf_hsa_shape* shape, const uint8_t* q8, const uint8_t* k8,
                                   const float* q_scale, const float* k_scale, const uint16_t* v,
                                   const int32_t* block_list, const int32_t* block_count, int32_t list_cap,
                                   float softmax_scale, uint16_t* out, int32_t tail_pieces, void* workspace,
                                   int64_t workspace_bytes, void* stream)
{
    Derived d;
    lf_status st = check_shape(shape, &d);
    if (st != LF_OK) return st;
    if (d.D != 128) return LF_ERR_SHAPE;
    if (list_cap < 0) return LF_ERR_CAP;
    if (!(softmax_scale == softmax_scale) || std::isinf(softmax_scale)) return LF_ERR_ARG;
    if (tail_pieces < 0 || workspace_bytes < 0) return LF_ERR_ARG;
    if (!q8 || !k8 || !q_scale || !k_scale || !v || !block_list || !block_count || !out) return LF_ERR_NULL;
    if (workspace_bytes > 0 && !workspace) return LF_ERR_NULL;
    if (!aligned16(q8) || !aligned16(k8) || !aligned16(q_scale) || !aligned16(k_scale) || !aligned16(v) ||
        !aligned16(block_list) || !aligned16(block_count) || !aligned16(out) ||
        (workspace_bytes > 0 && !aligned16(workspace)))
        return LF_ERR_ALIGN;
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return LF_ERR_NO_DEVICE;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return LF_ERR_NO_DEVICE;
    if (major != 10 || minor != 0) return LF_ERR_NO_DEVICE;
    int* err = nullptr;
    if ((st = error_word(&err)) != LF_OK) return st;
    const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(d.D));
    const long long BH = static_cast<long long>(d.B) * d.H;
    lf::AttnMaps m;
    const long long q_rows = BH * d.Lq, kv_rows = BH * d.kv_stride;
    if (!encode_rows_u8(&m.q, q8, q_rows, 64) || !encode_rows_u8(&m.q_rem, q8, q_rows, d.rem) ||
        !encode_rows_u8(&m.k, k8, kv_rows, 64) || !encode_rows_u8(&m.k_rem, k8, kv_rows, d.rem))
        return LF_ERR_CUDA;
    const bool v_il = d.F % 8 == 0 && d.kv_stride % 8 == 0 && encode_blocks_il(&m.v, v, kv_rows, 8) &&
                      encode_blocks_il(&m.v_rem, v, kv_rows, d.rem / 8);
    if (!v_il && (!encode_rows(&m.v, v, kv_rows, d.D, 64) || !encode_rows(&m.v_rem, v, kv_rows, d.D, d.rem)))
        return LF_ERR_CUDA;
    const long long n_rows = BH * d.Rq;
    int tail = 0, pieces = 0;
    if (workspace_bytes > 0 && tail_pieces != 1) {
        int sm = 0;
        if ((st = sm_count(&sm)) != LF_OK) return st;
        split_plan(n_rows, sm, list_cap, tail_pieces, workspace_bytes / split_slot_bytes(d.D), &tail, &pieces);
    }
    float* part_o = static_cast<float*>(workspace);
    float* part_ml = pieces ? part_o + static_cast<long long>(tail) * pieces * 64 * d.D : nullptr;
    lf::AttnArgs a{block_list, block_count, out, list_cap, d.Rq, d.bpf, d.F, d.Lq, d.Nkv, d.rem, d.kv_stride,
                   scale * 1.4426950408889634f, err, static_cast<int>(n_rows - tail), pieces, part_o, part_ml,
                   static_cast<int>(n_rows), static_cast<int>(n_rows - tail + static_cast<long long>(tail) * pieces),
                   q_scale, k_scale};
    return launch_status(lf::launch_attn_fp8(m, a, v_il, static_cast<cudaStream_t>(stream)));
}

lf_status lf_cag_budget(int32_t n_chunks, const double* T, const double* flops_w, double s_base, double s_target,
                        int32_t target_over_all, double* s_out, double* beta_out)
{
    if (!T || !s_out || !beta_out) return LF_ERR_NULL;
    if (n_chunks < 2) return LF_ERR_ARG;
    if (!(s_base >= 0.0 && s_base < 1.0) || !(s_target >= 0.0 && s_target < 1.0)) return LF_ERR_ARG;
    double W = 0.0, Wg = 0.0, Wa = 0.0;
    for (int i = 0; i < n_chunks; ++i) {
        const double w = flops_w ? flops_w[i] : static_cast<double>(i + 1);
        if (!(T[i] > 0.0) || !(w > 0.0) || std::isinf(T[i]) || std::isinf(w)) return LF_ERR_ARG;
        if (i == 0) {
            if (target_over_all) W += w;  // the dense first chunk counts in the budget
            continue;
        }
        const double alpha = 1.0 / std::sqrt(T[i]);
        W += w;
        Wg += w;
        Wa += w * alpha;
    }
    // sum_{i>1} w_i (s_base - alpha_i beta) = s_target * W, linear in beta.
    const double beta = (s_base * Wg - s_target * W) / Wa;
    *beta_out = beta;
    s_out[0] = 0.0;
    bool feasible = beta >= 0.0;
    for (int i = 1; i < n_chunks; ++i) {
        s_out[i] = s_base - beta / std::sqrt(T[i]);
        if (!(s_out[i] >= 0.0 && s_out[i] < 1.0)) feasible = false;
    }
    return feasible ? LF_OK : LF_ERR_INFEASIBLE;
}

int32_t lf_blocks_for_sparsity(double s, int32_t n_kv_blocks, int32_t n_sel_frames, int32_t bpf)
{
    if (!(s >= 0.0 && s < 1.0) || n_kv_blocks < 1 || n_sel_frames < 1 || bpf < 1) return -1;
    double x = std::floor((1.0 - s) * static_cast<double>(n_kv_blocks) / static_cast<double>(n_sel_frames) + 0.5);
    if (x < 1.0) x = 1.0;
    if (x > static_cast<double>(bpf)) x = static_cast<double>(bpf);
    return static_cast<int32_t>(x);
}

lf_status lf_get_device_error(int32_t* detail)
{
    int* p = nullptr;
    lf_status st = error_word(&p);
    if (st != LF_OK) return st;
    int h = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return LF_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&h, g_device_error, sizeof h) != cudaSuccess) return LF_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero) != cudaSuccess) return LF_ERR_CUDA;
    if (detail) *detail = h;
    if (h == 0) return LF_OK;
    return (h & lf::DEVERR_TIMEOUT) ? LF_ERR_DEVICE_TIMEOUT : LF_ERR_LIST;
}

}  // extern "C"

// ---- attention without allocation ---------------------------------------------
// The split's partial rows for lf_block_sparse_attn_static: a fixed array in the
// library image, so that callers that cannot allocate device memory need not.
static __device__ __align__(256) unsigned char g_attn_scratch[LF_ATTN_STATIC_SCRATCH_BYTES];

namespace {

void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_attn_scratch on the current device, looked up once per
// device at the first call and kept for the life of the process (host code
// cannot use the symbol itself as a device pointer). The kept address belongs
// to the device's primary context: after cudaDeviceReset it is stale, so a
// process that resets a device must not call lf_block_sparse_attn_static on it
// again (stated in lf_hsa.h).
lf_status static_scratch(void** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LF_ERR_NO_DEVICE;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_attn_scratch) != cudaSuccess || !p) return LF_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return LF_OK;
}

}  // namespace

extern "C" lf_status lf_block_sparse_attn_static(const lf_hsa_shape* shape, const uint16_t* q, const uint16_t* k,
                                                const uint16_t* v, const int32_t* block_list,
                                                const int32_t* block_count, int32_t list_cap,
                                                float softmax_scale, uint16_t* out, int32_t tail_pieces,
                                                void* stream)
{
    Derived d;
    lf_status st = check_shape(shape, &d);
    if (st != LF_OK) return st;
    if (list_cap < 0) return LF_ERR_CAP;
    if (!(softmax_scale == softmax_scale) || std::isinf(softmax_scale) || tail_pieces < 0) return LF_ERR_ARG;
    if (!q || !k || !v || !block_list || !block_count || !out) return LF_ERR_NULL;
    // scratch the split needs: the same plan lf_block_sparse_attn_ws makes
    long long need = 0;
    if (tail_pieces != 1) {
        int sm = 0;
        if ((st = sm_count(&sm)) != LF_OK) return st;
        int t = 0, kp = 0;
        split_plan(static_cast<long long>(d.B) * d.H * d.Rq, sm, list_cap, tail_pieces, -1, &t, &kp);
        need = static_cast<long long>(t) * kp * split_slot_bytes(d.D);
    }
    if (need > LF_ATTN_STATIC_SCRATCH_BYTES) return LF_ERR_SCRATCH;
    void* ws = nullptr;
    if (need > 0 && (st = static_scratch(&ws)) != LF_OK) return st;
    return lf_block_sparse_attn_ws(shape, q, k, v, block_list, block_count, list_cap, softmax_scale, out,
                                   need > 0 ? tail_pieces : 1, ws, need, stream);
}
