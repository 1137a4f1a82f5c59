/*
 * lf_hsa.h -- C ABI of the B200 (sm_100a) Light Forcing Hierarchical Sparse
 * Attention (HSA) library, liblf_hsa.so.
 *
 * One HSA attention call of a chunked autoregressive video diffusion
 * transformer, as described in "Light Forcing：通过稀疏注意力加速自回归视频扩散"
 * (paper.rainbus.top, execution-flow paragraph, stages 2 and 3) and
 * "Light Forcing: Accelerating Autoregressive Video Diffusion via Sparse
 * Attention" (gist.science, Technical Summary 2.2):
 *
 *   lf_pool              block mean pooling of q and k, frame mean pooling of k
 *   lf_pool_range        the same for a range of KV frames (pooled-key cache)
 *   lf_select_frames     per query block: frame scores, top-k memory frames T_r
 *                        plus the always-kept sink / recent / current frames
 *   lf_select_blocks     per selected frame: block scores, top-k blocks J_r(tau),
 *                        written as a compacted block list (the mask B_r)
 *   lf_select_mask       both selection levels in one launch
 *   lf_select_blocks_1d  one-dimensional variant: global block top-k over all
 *                        KV blocks, no frame level (the ablation baseline)
 *   lf_frame_index_build / lf_select_frames_ivf  coarse frame retrieval: a
 *                        k-means index over the frame means, probed per query
 *                        block (for very long videos)
 *   lf_block_sparse_attn softmax attention of each query block over the valid
 *                        tokens of its listed KV blocks (tcgen05 tensor cores)
 *   lf_block_sparse_attn_ws  the same with the last, partial wave of query
 *                        blocks split into list pieces (caller workspace)
 *   lf_attn_split_plan   that split's plan and workspace size (host only)
 *   lf_block_sparse_attn_static  the split attention for callers that cannot
 *                        allocate: its scratch is an array inside the library
 *   lf_quant_fp8_rows    per-token e4m3 codes and scales (the FP8 attention's q, k)
 *   lf_block_sparse_attn_fp8  the attention with e4m3 q and k (tcgen05 kind::f8f6f4)
 *
 * plus the host-side Chunk-Aware Growth budget solver (same pages, stage 1 /
 * Technical Summary 2.1).
 *
 * Conventions shared by every device entry point
 * ----------------------------------------------
 * - Layout: q and out are [batch, heads, n_cur*frame_tokens, head_dim] bf16,
 *   contiguous. k and v are [batch, heads, kv_stride, head_dim] bf16: head
 *   (b,h) starts at token (b*heads + h) * kv_stride and its first
 *   n_frames*frame_tokens tokens are the call's KV frames, in the order
 *   [sink frames][memory frames][recent frames][current-chunk frames].
 *   Queries are the current-chunk frames.
 * - Blocks are block_tokens = 64 consecutive tokens of one frame; a frame of F
 *   tokens has bpf = ceil(F/64) blocks and its last block may be partial (it
 *   holds F - 64*(bpf-1) tokens). Query block r = f*bpf + j is block j of
 *   current-chunk frame f (Rq = n_cur*bpf blocks); KV block g = tau*bpf + j is
 *   block j of KV frame tau (Nkv = n_frames*bpf blocks).
 * - bf16 data is passed as uint16_t bit patterns; pooled data is fp32.
 * - Ownership: the caller allocates every device buffer (inputs, outputs and
 *   the intermediate pooled / selection buffers, the split's workspace);
 *   lf_block_sparse_attn_static uses a fixed scratch array compiled into the
 *   library instead. The library never allocates,
 *   frees or synchronises; each call only enqueues kernels on `stream`
 *   (a cudaStream_t; NULL = the legacy default stream) and returns.
 * - Device pointers must be 16-byte aligned (the attention kernel reads them
 *   with TMA). Arguments are validated before anything is launched; a failed
 *   validation launches nothing.
 * - Device-side faults that only the kernel can see (an out-of-range block id
 *   in a list, a bounded wait that expired) never trap: the kernel records a
 *   code in a per-device error word and returns; lf_get_device_error() reads
 *   and clears it.
 */
#ifndef LF_HSA_H
#define LF_HSA_H

#include <stdint.h>

#if defined(__GNUC__)
#define LF_API __attribute__((visibility("default")))
#else
#define LF_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum lf_status {
    LF_OK = 0,
    LF_ERR_NULL = 1,           /* a required pointer is NULL */
    LF_ERR_ALIGN = 2,          /* a device pointer is not 16-byte aligned */
    LF_ERR_SHAPE = 3,          /* sizes outside the supported set (see lf_hsa_shape) */
    LF_ERR_TOPK = 4,           /* a top-k count below 1 */
    LF_ERR_CAP = 5,            /* list_cap smaller than the list the call writes */
    LF_ERR_INFEASIBLE = 6,     /* CAG: beta < 0 or some s_i outside [0, 1) */
    LF_ERR_CUDA = 7,           /* a CUDA runtime / launch call failed */
    LF_ERR_DEVICE_TIMEOUT = 8, /* device error word: a bounded wait in a kernel expired */
    LF_ERR_ARG = 9,            /* another invalid scalar (chunk index, sparsity, scale) */
    LF_ERR_LIST = 10,          /* device error word: a block id or count out of range */
    LF_ERR_NO_DEVICE = 11,     /* no usable sm_100 device */
    LF_ERR_SCRATCH = 12        /* the call needs more than the library's static scratch array */
} lf_status;

/*
 * Sizes of one HSA call.
 *   batch, heads >= 1; head_dim in {64, 128}; block_tokens == 64;
 *   1 <= frame_tokens <= 8192 (so bpf <= 128);
 *   n_sink, n_recent >= 0, n_cur >= 1, n_sink + n_recent + n_cur <= n_frames;
 *   the number of memory frames n_frames - n_sink - n_recent - n_cur <= 1024;
 *   kv_stride = 0 means n_frames*frame_tokens, otherwise >= that.
 */
typedef struct lf_hsa_shape {
    int32_t batch;
    int32_t heads;
    int32_t head_dim;
    int32_t frame_tokens;
    int32_t block_tokens;
    int32_t n_frames;
    int32_t n_sink;
    int32_t n_recent;
    int32_t n_cur;
    int64_t kv_stride;
} lf_hsa_shape;

/*
 * Token compression (paper.rainbus.top, execution flow, stage 2; gist.science
 * Technical Summary 2.2 "Token Compression").
 *   q_pool  [B,H,Rq,D]  fp32: mean of the tokens of each query block
 *   k_pool  [B,H,Nkv,D] fp32: mean of the tokens of each KV block
 *   k_frame [B,H,NF,D]  fp32: mean of all tokens of each KV frame (k^ of the
 *                              memory frames is the slice [n_sink, n_sink+n_mem))
 * Partial blocks are averaged over their real tokens. Reads q and k once.
 * Errors: LF_ERR_NULL, LF_ERR_ALIGN, LF_ERR_SHAPE, LF_ERR_CUDA.
 */
LF_API lf_status lf_pool(const lf_hsa_shape* shape, const uint16_t* q, const uint16_t* k,
                  float* q_pool, float* k_pool, float* k_frame, void* stream);

/*
 * Token compression of a range of KV frames only: writes the k_pool rows and
 * k_frame entries of frames [frame_begin, frame_end) (same layouts as lf_pool;
 * every other entry is left untouched) and, when pool_q != 0, all of q_pool.
 * Past KV frames do not change while a chunk denoises, so a caller that keeps
 * k_pool / k_frame between calls of the same shape re-pools only the frames
 * that changed (the current chunk) -- the pooled values are identical to a
 * full lf_pool of the same k (per frame, the same arithmetic in the same
 * order). The pages state that retrieval costs about 2 % of the run as history
 * grows (paper.rainbus.top, limitations and conclusion); this is the persistent
 * pooled-key cache that keeps the per-call pooling cost independent of the
 * history length. Pointers, layouts and ownership as lf_pool; q may be NULL
 * when pool_q == 0. Errors: LF_ERR_NULL, LF_ERR_ALIGN, LF_ERR_SHAPE,
 * LF_ERR_ARG (0 <= frame_begin <= frame_end <= n_frames violated), LF_ERR_CUDA.
 */
LF_API lf_status lf_pool_range(const lf_hsa_shape* shape, const uint16_t* q, const uint16_t* k,
                        int32_t frame_begin, int32_t frame_end, int32_t pool_q,
                        float* q_pool, float* k_pool, float* k_frame, void* stream);

/* Number of frames in each T_r: n_frames when chunk_index == 1, else
 * n_sink + min(topk_frames, n_mem) + n_recent + n_cur. Returns -1 on a bad shape. */
LF_API int32_t lf_frames_selected(const lf_hsa_shape* shape, int32_t chunk_index, int32_t topk_frames);

/*
 * Frame-level selection (paper.rainbus.top, execution flow, stage 3, first
 * level: p_r = <q~_r, k^_M>, top-k frames T_r, sink / most recent / current
 * chunk frames always kept; gist.science Technical Summary 2.2 "Frame
 * Selection").
 *   chunk_index  1-based position of the chunk in the rollout; chunk 1 is
 *                dense (stage 1) and selects every frame.
 *   topk_frames  k_f >= 1; values above n_mem keep every memory frame.
 *   frame_sel    [B,H,Rq,n_sel] int32 out, n_sel = lf_frames_selected(...):
 *                the frame ids of T_r in ascending order.
 * Scores are fp32 inner products; among equal scores the lower frame id wins.
 * Errors: LF_ERR_NULL, LF_ERR_ALIGN, LF_ERR_SHAPE, LF_ERR_TOPK, LF_ERR_ARG,
 * LF_ERR_CUDA.
 */
LF_API lf_status lf_select_frames(const lf_hsa_shape* shape, int32_t chunk_index, int32_t topk_frames,
                           const float* q_pool, const float* k_frame, int32_t* frame_sel,
                           void* stream);

/* Length of each block list row: n_sel * min(topk_blocks, bpf) (n_frames*bpf
 * for chunk 1). Returns -1 on a bad shape. */
LF_API int32_t lf_list_capacity(const lf_hsa_shape* shape, int32_t chunk_index, int32_t topk_frames,
                         int32_t topk_blocks);

/*
 * Block-level selection (paper.rainbus.top, execution flow, stage 3, second
 * level: o_r(tau,j) = <q~_r, k~_j^(tau)>, top-k blocks J_r(tau) inside each
 * selected frame, mask B_r(tau,j) = 1[tau in T_r, j in J_r(tau)];
 * gist.science Technical Summary 2.2 "Block Selection").
 *   frame_sel    [B,H,Rq,n_sel] int32 from lf_select_frames (same chunk_index
 *                and topk_frames).
 *   topk_blocks  k_b >= 1; values above bpf keep every block of a frame.
 *   block_list   [B,H,Rq,list_cap] int32 out: row (b,h,r) holds the global KV
 *                block ids tau*bpf + j of the mask, frame by frame in the order
 *                of frame_sel and ascending j inside a frame (so the row is
 *                ascending when frame_sel is). Entries past the count are not
 *                written.
 *   block_count  [B,H,Rq] int32 out: n_sel * min(topk_blocks, bpf) per row
 *                (every row keeps the same number of blocks).
 *   list_cap     >= lf_list_capacity(...), else LF_ERR_CAP.
 * Among equal scores the lower block index wins.
 * Errors: LF_ERR_NULL, LF_ERR_ALIGN, LF_ERR_SHAPE, LF_ERR_TOPK, LF_ERR_CAP,
 * LF_ERR_ARG, LF_ERR_CUDA.
 */
LF_API lf_status lf_select_blocks(const lf_hsa_shape* shape, int32_t chunk_index, int32_t topk_frames,
                           int32_t topk_blocks, const float* q_pool, const float* k_pool,
                           const int32_t* frame_sel, int32_t* block_list, int32_t* block_count,
                           int32_t list_cap, void* stream);

/*
 * Both levels of the mask selection in one launch: lf_select_frames followed by
 * lf_select_blocks (same passages, arguments, layouts and errors), computed per
 * query block by one CTA (frames, then the blocks of the selected frames) with
 * the same arithmetic, so frame_sel, block_list and block_count are
 * bit-identical to the two separate calls.
 */
LF_API lf_status lf_select_mask(const lf_hsa_shape* shape, int32_t chunk_index, int32_t topk_frames,
                         int32_t topk_blocks, const float* q_pool, const float* k_frame,
                         const float* k_pool, int32_t* frame_sel, int32_t* block_list,
                         int32_t* block_count, int32_t list_cap, void* stream);

/*
 * One-dimensional (single-granularity) block selection: the variant without
 * the frame level that the ablation of "南洋理工大学打造视频生成新引擎"
 * (163.com, section 4) compares against. Reading (the pages name the variant
 * without spelling it out): o_r(g) = <q~_r, k~_g> for every KV block g of the
 * call, the row keeps the top-k of them with no frame forced in.
 *   k_pool       [B,H,Nkv,D] fp32 from lf_pool (q_pool likewise).
 *   topk_blocks  k >= 1; k >= Nkv, or chunk_index == 1 (dense first chunk),
 *                keeps every block.
 *   block_list   [B,H,Rq,list_cap] int32 out: the kept global block ids,
 *                ascending; block_count [B,H,Rq] out: min(k, Nkv) (Nkv for
 *                chunk 1). The lists feed lf_block_sparse_attn unchanged.
 * Among equal scores the lower block index wins. Nkv is limited to 16384.
 * Errors: LF_ERR_NULL, LF_ERR_ALIGN, LF_ERR_SHAPE (also Nkv > 16384),
 * LF_ERR_TOPK, LF_ERR_CAP (list_cap below the kept count), LF_ERR_ARG
 * (chunk_index < 1), LF_ERR_NO_DEVICE, LF_ERR_CUDA. The kernel streams k_pool
 * through shared memory with bulk copies whose waits are bounded (1 s); a wait
 * that expires sets the device error word (lf_get_device_error) and the row's
 * list is left unwritten.
 */
LF_API lf_status lf_select_blocks_1d(const lf_hsa_shape* shape, int32_t chunk_index, int32_t topk_blocks,
                              const float* q_pool, const float* k_pool, int32_t* block_list,
                              int32_t* block_count, int32_t list_cap, void* stream);

/*
 * Coarse frame retrieval for very long videos: an index over the frame means.
 * "Light Forcing：通过稀疏注意力加速自回归视频扩散" (paper.rainbus.top,
 * weaknesses paragraph, point 2) notes that the frame candidates grow linearly
 * with the video and names a hierarchical index as the remedy without fixing
 * it. Reading taken: per (batch, head), k-means with squared L2 distance over
 * the memory-frame means k^_m (the slice [n_sink, n_sink + n_mem) of k_frame),
 * C = min(n_clusters, n_mem) clusters started at memory frames floor(i*n_mem/C),
 * Lloyd rounds until no assignment changes or `iters` updates were made (then
 * one last assignment); an empty cluster keeps its centroid; equal distances go
 * to the lower cluster. Computed in fp64 from the fp32 frame means. Build it
 * once per head and again when frames are appended (it does not depend on q).
 *   n_clusters  1..64; iters 0..100000.
 *   centroids   [B,H,n_clusters,D] fp32 out (rows [0, C) written)
 *   labels      [B,H,max(n_mem,1)] int32 out: the cluster of each memory frame
 *   offsets     [B,H,n_clusters+1] int32 out: cluster j holds
 *               members[offsets[j] .. offsets[j+1])
 *   members     [B,H,max(n_mem,1)] int32 out: memory-frame indices (0-based in
 *               M) grouped by cluster, ascending within a cluster
 * One CTA per (batch, head). All pointers 16-byte aligned.
 * Errors: LF_ERR_NULL, LF_ERR_ALIGN, LF_ERR_SHAPE, LF_ERR_ARG, LF_ERR_CUDA.
 */
LF_API lf_status lf_frame_index_build(const lf_hsa_shape* shape, int32_t n_clusters, int32_t iters,
                               const float* k_frame, float* centroids, int32_t* labels,
                               int32_t* offsets, int32_t* members, void* stream);

/*
 * Frame-level selection through the index of lf_frame_index_build (same
 * passages). Per query block: clusters ordered by <q~_r, c_j> (equal scores:
 * lower cluster first); the best n_probe are probed, and further ones in that
 * order until the probed clusters hold min(topk_frames, n_mem) frames; T_r is
 * the exact top-k of the probed clusters' frames by p_r = <q~_r, k^_m> (equal
 * scores: lower frame) plus the sink, recent and current-chunk frames,
 * ascending, in the layout of lf_select_frames (lf_select_blocks consumes it
 * unchanged). With every cluster probed the result is lf_select_frames' result
 * (same fp32 scores). chunk_index == 1 selects every frame.
 *   n_clusters  the value given to lf_frame_index_build; n_probe >= 1.
 * Errors: LF_ERR_NULL, LF_ERR_ALIGN, LF_ERR_SHAPE, LF_ERR_TOPK, LF_ERR_ARG,
 * LF_ERR_CUDA.
 */
LF_API lf_status lf_select_frames_ivf(const lf_hsa_shape* shape, int32_t chunk_index, int32_t topk_frames,
                               int32_t n_clusters, int32_t n_probe, const float* q_pool,
                               const float* k_frame, const float* centroids, const int32_t* offsets,
                               const int32_t* members, int32_t* frame_sel, void* stream);

/*
 * Per-token e4m3 quantisation for the FP8 attention (lf_block_sparse_attn_fp8).
 * The pages put FP8 with per-token activation scales on the model's linear
 * layers ("南洋理工大学打造视频生成新引擎", 163.com, deployment section;
 * gist.science, Technical Summary 4) and describe no FP8 attention; reading taken
 * here: Q and K quantised per token (one scale per row of head_dim values).
 *   x       [n_rows, head_dim] bf16 (e.g. q, or k with its head stride padding)
 *   x8      [n_rows, head_dim] uint8 out: e4m3 codes (OCP E4M3: bias 7, 3 mantissa
 *           bits, largest finite 448)
 *   scales  [n_rows] fp32 out: s = fl32(amax / 448) (1 for an all-zero row)
 * code = e4m3(fl32(x / s)) with IEEE fp32 division, round to nearest even,
 * saturating at 448; x is about s * code. One warp per row.
 * Errors: LF_ERR_NULL, LF_ERR_ALIGN, LF_ERR_ARG (head_dim not 64 or 128, n_rows
 * < 0), LF_ERR_SHAPE, LF_ERR_CUDA.
 */
LF_API lf_status lf_quant_fp8_rows(const uint16_t* x, int64_t n_rows, int32_t head_dim, uint8_t* x8,
                            float* scales, void* stream);

/*
 * Block-sparse softmax attention (paper.rainbus.top, execution flow, stage 3,
 * final step: attention over the block mask).
 *   out[b,h,t,:] = sum_s softmax_s(scale * <q_t, k_s>) v_s over every valid
 *   token s of the KV blocks listed for t's query block (no causal mask).
 *   block_list / block_count as written by lf_select_blocks (any order, no
 *   duplicates expected); list_cap is the row stride of block_list.
 *   softmax_scale <= 0 selects 1/sqrt(head_dim).
 *   out [B,H,Lq,D] bf16: every valid query row is written; a row whose list is
 *   empty gets zeros.
 * Block ids outside [0, Nkv) or counts outside [0, list_cap] are skipped /
 * clamped on the device and reported as LF_ERR_LIST by lf_get_device_error().
 * Errors: LF_ERR_NULL, LF_ERR_ALIGN, LF_ERR_SHAPE, LF_ERR_CAP, LF_ERR_ARG,
 * LF_ERR_NO_DEVICE, LF_ERR_CUDA.
 */
LF_API lf_status lf_block_sparse_attn(const lf_hsa_shape* shape, const uint16_t* q, const uint16_t* k,
                               const uint16_t* v, const int32_t* block_list,
                               const int32_t* block_count, int32_t list_cap, float softmax_scale,
                               uint16_t* out, void* stream);

/*
 * lf_block_sparse_attn with the last, partial wave split (same passage; the
 * split is a scheduling choice and changes the result only by fp32 rounding).
 * One CTA computes one query block; with n_rows = B*H*Rq query blocks on a
 * device of sm SMs the last r = n_rows mod sm of them (all of them when
 * n_rows < sm) would run alone on r SMs. Their lists are cut into `pieces`
 * consecutive pieces, each piece's softmax partial (normalised rows plus the
 * row max and denominator) goes to `workspace`, and a second kernel merges
 * the pieces of each row exactly as the online softmax would.
 *   tail_pieces      0: automatic plan (lf_attn_split_plan on the current
 *                    device); 1: no split; >= 2: that many pieces per list.
 *                    The piece count is lowered to what `workspace` holds and
 *                    to list_cap; below 2 nothing is split. (This entry point
 *                    caps the pieces at its workspace; lf_block_sparse_attn_static,
 *                    whose scratch is fixed, refuses a split that does not fit.)
 *   workspace        device scratch, 16-byte aligned, owned by the caller,
 *                    64 * (head_dim + 2) * 4 bytes per piece slot (r * pieces
 *                    slots); NULL with workspace_bytes == 0 means no split.
 *                    Two calls in flight at once need two workspaces.
 * Enqueues two kernels when it splits, one otherwise.
 * Errors: those of lf_block_sparse_attn; LF_ERR_ARG for tail_pieces < 0 or
 * workspace_bytes < 0; LF_ERR_NULL / LF_ERR_ALIGN for the workspace.
 */
LF_API lf_status lf_block_sparse_attn_ws(const lf_hsa_shape* shape, const uint16_t* q, const uint16_t* k,
                                  const uint16_t* v, const int32_t* block_list,
                                  const int32_t* block_count, int32_t list_cap, float softmax_scale,
                                  uint16_t* out, int32_t tail_pieces, void* workspace,
                                  int64_t workspace_bytes, void* stream);

/*
 * The automatic split plan of lf_block_sparse_attn_ws, host only.
 *   sm               SM count to plan for; <= 0 queries the current device
 *                    (LF_ERR_NO_DEVICE without one).
 *   tail_rows out    query blocks whose lists are split (0: no split)
 *   pieces out       pieces per split list: min(sm / tail_rows, list_cap / 8);
 *                    0 (no split) when sm / tail_rows < 8 (the last wave
 *                    fills more than an eighth of the SMs) or the minimum is
 *                    below 2
 *   workspace_bytes out  tail_rows * pieces * 64 * (head_dim + 2) * 4
 * Errors: LF_ERR_NULL, LF_ERR_SHAPE, LF_ERR_CAP, LF_ERR_NO_DEVICE.
 */
LF_API lf_status lf_attn_split_plan(const lf_hsa_shape* shape, int32_t list_cap, int32_t sm,
                             int32_t* tail_rows, int32_t* pieces, int64_t* workspace_bytes);

/* Size of the scratch array behind lf_block_sparse_attn_static. */
#define LF_ATTN_STATIC_SCRATCH_BYTES (8ll << 20)

/*
 * lf_block_sparse_attn_ws for callers that cannot allocate device memory.
 * The paper has no counterpart: this is a packaging of the same computation.
 * Some callers have no way to allocate: a plug-in inside a host application
 * that owns the whole device-memory budget and hands out no allocator, or a
 * loop that must not call cudaMalloc / cudaFree because they synchronise the
 * device and may fail once the budget is spent. Such a caller passes only its
 * inputs and outputs; the split's partial rows go to a scratch array of
 * LF_ATTN_STATIC_SCRATCH_BYTES (8 MiB) compiled into this library, which every
 * GPU that loads the library holds until the process exits. The call
 * allocates nothing.
 *   tail_pieces  as in lf_block_sparse_attn_ws (0: automatic plan, 1: no
 *                split, >= 2: that many pieces per split list).
 * Set-up: the first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and keeps it; make that
 * first call before any stream capture. The kept address belongs to the
 * device's primary context: a process that calls cudaDeviceReset must not call
 * this entry point on that device afterwards.
 * Sharing: every call on a device uses the same array and leaves its partial
 * rows in it. Each call writes every slot it reads before reading it, so
 * nothing has to start at zero, but two calls that overlap on the GPU (other
 * streams, other threads) race on the array and give wrong results: order them.
 * Errors: those of lf_block_sparse_attn_ws; LF_ERR_SCRATCH (nothing launched)
 * when the split would need more than LF_ATTN_STATIC_SCRATCH_BYTES, i.e. more
 * than LF_ATTN_STATIC_SCRATCH_BYTES / (64 * (head_dim + 2) * 4) piece slots
 * (the automatic plan uses at most one slot per SM: 148 of 252 at head_dim 128).
 */
LF_API lf_status lf_block_sparse_attn_static(const lf_hsa_shape* shape, const uint16_t* q, const uint16_t* k,
                                      const uint16_t* v, const int32_t* block_list,
                                      const int32_t* block_count, int32_t list_cap,
                                      float softmax_scale, uint16_t* out, int32_t tail_pieces,
                                      void* stream);

/*
 * Block-sparse attention with e4m3 queries and keys (head_dim 128): the FP8
 * attention of this library. Same passage and mask as lf_block_sparse_attn; the
 * FP8 reading is lf_quant_fp8_rows'. Scores are <q8, k8> (exact e4m3 products,
 * fp32 accumulation on the tensor cores, kind::f8f6f4) times q_scale(row) *
 * k_scale(key); the softmax is fp32 as in the bf16 path and P and V stay bf16.
 *   q8       [B,H,Lq,128] uint8 e4m3 codes, q_scale [B,H,Lq] fp32
 *   k8       [B,H,kv_stride,128] uint8 e4m3 codes, k_scale [B,H,kv_stride] fp32
 *   v        [B,H,kv_stride,128] bf16
 *   the rest as lf_block_sparse_attn_ws (list, scale, out, split and workspace).
 * Errors: those of lf_block_sparse_attn_ws; LF_ERR_SHAPE when head_dim != 128.
 */
LF_API lf_status lf_block_sparse_attn_fp8(const lf_hsa_shape* shape, const uint8_t* q8, const uint8_t* k8,
                                   const float* q_scale, const float* k_scale, const uint16_t* v,
                                   const int32_t* block_list, const int32_t* block_count, int32_t list_cap,
                                   float softmax_scale, uint16_t* out, int32_t tail_pieces,
                                   void* workspace, int64_t workspace_bytes, void* stream);

/*
 * Chunk-Aware Growth budget solver, host only, fp64 (paper.rainbus.top,
 * execution flow, stage 1; gist.science Technical Summary 2.1; 163.com
 * article section 2).
 *   s_1 = 0 (first chunk dense); s_i = s_base - alpha_i * beta for i > 1 with
 *   alpha_i = 1/sqrt(T[i-1]); beta solves
 *       sum_i w_i s_i = s_target * sum_i w_i
 *   over all chunks (target_over_all != 0) or over chunks 2..n (== 0).
 *   flops_w = NULL uses w_i = i (dense attention FLOPs of chunk i when the KV
 *   length grows by one chunk per step).
 *   s_out[n_chunks] and *beta_out are written whenever the arguments are valid,
 *   also when the result is infeasible.
 * Errors: LF_ERR_NULL, LF_ERR_ARG (n_chunks < 2, a T or w <= 0, s outside
 * [0,1)), LF_ERR_INFEASIBLE (beta < 0 or some s_i outside [0,1)).
 */
LF_API lf_status lf_cag_budget(int32_t n_chunks, const double* T, const double* flops_w, double s_base,
                        double s_target, int32_t target_over_all, double* s_out,
                        double* beta_out);

/*
 * Per-frame block count for a target block sparsity s in [0,1): the kept
 * (1 - s) * n_kv_blocks blocks spread evenly over n_sel selected frames,
 * rounded to nearest and clamped to [1, bpf]. The pages give no formula for
 * this step; this is the plainest reading. Returns -1 on invalid arguments.
 */
LF_API int32_t lf_blocks_for_sparsity(double s, int32_t n_kv_blocks, int32_t n_sel_frames, int32_t bpf);

/* Reads and clears the error word of the current device: LF_OK or
 * LF_ERR_DEVICE_TIMEOUT / LF_ERR_LIST. Synchronises the current device. */
LF_API lf_status lf_get_device_error(int32_t* detail);

/* Static description of a status code. */
LF_API const char* lf_status_string(lf_status status);

/* Library version, e.g. "lf_hsa 0.1.0 sm_100a". */
LF_API const char* lf_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LF_HSA_H */
