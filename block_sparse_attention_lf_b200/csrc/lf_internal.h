// lf_internal.h -- launch interfaces between the C ABI layer (lf_api.cu) and
// the kernel translation units. Not part of the public ABI.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace lf {

struct PoolArgs {
    const uint16_t* q;
    const uint16_t* k;
    float* q_pool;
    float* k_pool;
    float* k_frame;
    int BH, D, F, bpf, NF, n_cur;
    long long kv_stride;  // tokens between heads in k
    int f0, nk;           // KV frames [f0, f0 + nk) are pooled
    int pool_q;           // also pool the query frames
    int* err;             // device error word (an expired bounded wait)
};

struct SelectFramesArgs {
    const float* q_pool;
    const float* k_frame;
    int* frame_sel;
    int BH, D, Rq, NF, n_sink, n_recent, n_cur, n_sel, topk, chunk_index;
};

struct SelectBlocksArgs {
    const float* q_pool;
    const float* k_pool;
    const int* frame_sel;
    int* block_list;
    int* block_count;
    int BH, D, Rq, NF, bpf, n_sel, kb, list_cap, chunk_index;
    int* err;
};

// One-dimensional (single-granularity) block selection: every KV block of the
// head is a candidate; the row keeps the top `kb` of them.
struct SelectBlocks1dArgs {
    const float* q_pool;
    const float* k_pool;
    int* block_list;
    int* block_count;
    int BH, D, Rq, Nkv, kb, list_cap, chunk_index;
    int* err;  // device error word (bounded waits of the bulk-copy ring)
};

constexpr int SEL1D_MAX_NKV = 16384;  // candidate scores held in shared memory (64 KB per scored row)

// Coarse frame retrieval: a k-means index over each head's memory-frame means.
constexpr int IVF_MAX_CLUSTERS = 64;
constexpr int IVF_MAX_MEM = 1024;  // memory frames per call (the shape limit)

struct FrameIndexArgs {
    const float* k_frame;  // [BH, NF, D]
    float* centroids;      // [BH, C_stride, D]: rows [0, C) written
    int* labels;           // [BH, m_stride]: cluster of each memory frame
    int* offsets;          // [BH, C_stride + 1]: members of cluster j are members[offsets[j], offsets[j+1])
    int* members;          // [BH, m_stride]: memory-frame indices grouped by cluster, ascending in a cluster
    int BH, D, NF, n_sink, n_mem, C, C_stride, m_stride, iters;
};

struct SelectFramesIvfArgs {
    const float* q_pool;
    const float* k_frame;
    const float* centroids;
    const int* offsets;
    const int* members;
    int* frame_sel;
    int BH, D, Rq, NF, n_sink, n_recent, n_cur, n_mem, n_sel, topk, chunk_index, C, C_stride, m_stride, n_probe;
};

size_t frame_index_smem_bytes(int C, int n_mem, int D);

struct AttnArgs {
    const int* block_list;
    const int* block_count;
    uint16_t* out;
    int list_cap, Rq, bpf, F, Lq, Nkv, rem;
    long long kv_stride;
    float scale_log2;  // softmax scale * log2(e)
    int* err;
    // Split of the tail: query blocks [0, n_whole) are one work unit each; every
    // later query block's list is cut into `pieces` consecutive pieces, one unit
    // each, whose normalised fp32 partial rows and (stabiliser, sum) pairs go to
    // part_o / part_ml and are merged by a second kernel.
    int n_whole, pieces;  // pieces == 0: no split
    float* part_o;        // [slot][64][D]; slot = (query block - n_whole) * pieces + piece
    float* part_ml;       // [slot][64][2]: stabiliser (log2 units), softmax denominator
    int n_rows;           // query blocks of the call (B * H * Rq)
    int n_units;          // CTAs of the attention grid: n_whole whole lists + (n_rows - n_whole) * pieces pieces
    const float* q_scale;  // e4m3 path: per-token scales of q8 [B*H*Lq] and k8 [B*H*kv_stride]
    const float* k_scale;
};

struct AttnMaps {
    CUtensorMap q, q_rem, k, k_rem, v, v_rem;
};

cudaError_t launch_pool(const PoolArgs& a, cudaStream_t s);
cudaError_t launch_select_frames(const SelectFramesArgs& a, cudaStream_t s);
cudaError_t launch_select_blocks(const SelectBlocksArgs& a, cudaStream_t s);
// both selection levels in one launch (frame_sel and the block lists, as the two above)
cudaError_t launch_select_fused(const SelectFramesArgs& fa, const SelectBlocksArgs& ba, cudaStream_t s);
// per-row e4m3 codes and fp32 scales of n_rows rows of D bf16 values
cudaError_t launch_quant_rows(const uint16_t* x, long long n_rows, int D, uint8_t* x8, float* scale, cudaStream_t s);
cudaError_t launch_select_blocks_1d(const SelectBlocks1dArgs& a, cudaStream_t s);
cudaError_t launch_frame_index(const FrameIndexArgs& a, cudaStream_t s);
cudaError_t launch_select_frames_ivf(const SelectFramesIvfArgs& a, cudaStream_t s);
// interleaved: K/V tensor maps are the 4-D block maps (head_dim 128 only).
cudaError_t launch_attn(const AttnMaps& m, const AttnArgs& a, int D, bool interleaved, cudaStream_t s);
// e4m3 q/k (head_dim 128): maps q / q_rem / k / k_rem are uint8 row maps, v / v_rem bf16
// (4-D block maps when v_interleaved)
cudaError_t launch_attn_fp8(const AttnMaps& m, const AttnArgs& a, bool v_interleaved, cudaStream_t s);

}  // namespace lf
