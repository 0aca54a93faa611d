/*
 * dsa.h -- C ABI of the B200 (sm_100a) DeepSeek Sparse Attention hot path.
 *
 * The method (pages "一文讀懂DeepSeek-V3.2核心技術DSA", section "DSA 的四步工作流程";
 * "DeepSeek-V3.2加速技术详解", sections 3.1-3.2; "DeepSeek 稀疏注意力路线", section
 * "DeepSeek-V3.2：DSA / 两阶段流程") runs three steps per query token t:
 *   1. lightning indexer:  I[t,s] = sum_j w[t,j] * ReLU(q_I[t,j,:] . k_I[s,:])
 *      over the visible keys s <= pos_t, FP8 E4M3 queries/keys of 128 dims;
 *   2. fine-grained top-k: the k keys with the highest I (all of them when the
 *      context holds <= k keys);
 *   3. sparse MLA in MQA form: softmax attention of every query head over only
 *      the selected rows of the shared latent cache (576-dim key = 512 latent +
 *      64 RoPE; the value is the 512-dim latent).
 *
 * Conventions for every call
 *   - Pointers marked (device) are CUDA device pointers; everything else is host.
 *   - The caller owns every buffer and the stream.  The library allocates no
 *     device memory (workspaces are the caller's) and keeps no per-call state;
 *     it creates TMA descriptors on the host per call.  Kept per device across
 *     calls: cached kernel attributes, one cuBLASLt handle (created by the first
 *     dsa_project_append) and the fixed array of dsa_indexer_scores_noalloc;
 *     dsa_forward_host creates CUDA events for its cross-stream ordering and
 *     destroys them before it returns.  All calls are asynchronous on `stream`
 *     (a cudaStream_t passed as void*; NULL = the legacy default stream) and
 *     never synchronise, except dsa_read_device_status.
 *   - Arguments are checked on the host before any launch; on a failed check
 *     nothing is launched or written and the status says why.
 *   - Errors the host cannot see (a query position beyond its sequence, an index
 *     out of range, a bounded wait that ran out) are recorded as bit flags in a
 *     status word at the start of the workspace `ws`; each call clears the word
 *     when it starts.  Read it with dsa_read_device_status.
 *   - Batches: sequence b owns the cache rows kv_offset[b] .. kv_offset[b] +
 *     kv_len[b] - 1 of k_idx and kv (rows of one sequence are contiguous), or,
 *     with a paged layout (page_size > 0), key s of sequence b sits in cache row
 *     page_table[b * pages_per_seq + s / page_size] * page_size + s % page_size
 *     (the block-table layout of paged inference caches: a sequence's rows are
 *     contiguous only within a page).  Both k_idx and kv use the same rows.
 *     Query t belongs to sequence q_seq[t] and sees its keys 0 .. q_pos[t]
 *     (n_t = q_pos[t] + 1 keys; causal and inclusive).  Key and selection
 *     indices are local to the sequence.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DSA_ABI_VERSION 2

/* Fixed widths of the method (one indexer key per token of 128 dims; latent 512
 * + RoPE 64; value = latent). */
#define DSA_D_INDEX 128
#define DSA_D_QK 576
#define DSA_D_V 512

typedef enum dsa_status {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARGUMENT = 1,   /* null pointer, negative size, inconsistent sizes */
  DSA_ERR_UNSUPPORTED = 2,        /* a size outside the supported shapes below */
  DSA_ERR_WORKSPACE_TOO_SMALL = 3,/* ws_bytes < dsa_workspace_size(...) */
  DSA_ERR_CUDA = 4,               /* a CUDA runtime/driver call or launch failed */
  DSA_ERR_DEVICE = 5              /* dsa_read_device_status found a device flag */
} dsa_status;

/* Bit flags of the device status word. */
#define DSA_DEV_BAD_QUERY 1u      /* q_seq out of [0,B) or q_pos out of [0, kv_len) */
#define DSA_DEV_BAD_INDEX 2u      /* a selected index >= kv_len of its sequence */
#define DSA_DEV_TIMEOUT 4u        /* a bounded in-kernel wait expired; results invalid */
#define DSA_DEV_INTERNAL 8u       /* a kernel precondition failed (e.g. shared-memory alignment); results invalid */

typedef struct dsa_batch {
  int32_t num_seqs;        /* B >= 1 */
  int32_t num_q;           /* T >= 0 query tokens in this call */
  int32_t max_kv_len;      /* >= every kv_len[b]; sizes grids and score rows */
  int32_t max_q_per_seq;   /* >= the number of queries of any one sequence (a grouping hint
                              for the indexer); 0 means "unknown" (taken as num_q) */
  int64_t kv_rows;         /* rows held by the k_idx / kv buffers (>= kv_offset[b] + kv_len[b]) */
  const int64_t *kv_offset;/* (device) [B] first cache row of sequence b */
  const int32_t *kv_len;   /* (device) [B] cache rows of sequence b */
  const int32_t *q_seq;    /* (device) [T] sequence of query t */
  const int32_t *q_pos;    /* (device) [T] position of query t, 0 <= q_pos < kv_len */
  /* Paged layout (ABI 2).  page_size = 0: contiguous rows from kv_offset (the
   * fields below are ignored).  page_size > 0: a multiple of 64; kv_offset is
   * ignored (may be NULL); page_table (device) int32 [B, pages_per_seq] holds the
   * physical page of each page of a sequence, pages_per_seq * page_size >=
   * max_kv_len; kv_rows is the number of physical rows (pages * page_size).  A
   * page entry that points outside kv_rows raises DSA_DEV_BAD_INDEX and reads
   * as zeros. */
  int32_t page_size;
  int32_t pages_per_seq;
  const int32_t *page_table;
} dsa_batch;

/* Operation codes for dsa_workspace_size. */
#define DSA_OP_INDEXER 0
#define DSA_OP_TOPK 1
#define DSA_OP_SPARSE_MLA 2
#define DSA_OP_FORWARD 3
#define DSA_OP_PROJECT 4
#define DSA_OP_MLA_BACKWARD 5
#define DSA_OP_FORWARD_HOST 6

/*
 * Bytes of workspace `ws` an operation needs (always >= 256: the status word and
 * a small plan live at its start).  `ld` is the score row stride (elements) for
 * DSA_OP_FORWARD (0 = the default, max_kv_len rounded up to a multiple of 4).
 * Returns 0 for an invalid op or batch.
 */
size_t dsa_workspace_size(int op, const dsa_batch *batch, int H_I, int H, int k, int64_t ld);

/*
 * The step before the path ("四步工作流程" 第一步 查詢與鍵的投影: queries, keys and
 * per-head weights projected from the hidden states with rotary embeddings;
 * "DeepSeek 稀疏注意力路线", V3's MLA: the latent down-projection that is cached and
 * the decoupled RoPE channel): projections of the T new tokens, RoPE, storage casts
 * and cache append, with the caller's (e.g. synthetic) weights.
 *   hidden (device) bf16 bits [T, d_model]
 *   w_all  (device) bf16 bits [N, d_model], N = H_I*128 + 128 + H_I + 512 + 64 + H*576,
 *          stacked rows for: the indexer query heads (H_I x 128), the indexer key
 *          (128), the per-head weights (H_I), the latent (512), the RoPE key (64),
 *          the latent query heads (H x 512), the RoPE query heads (H x 64)
 *   Y = hidden W^T in fp32 (tensor cores, fp32 accumulation), then for token t at
 *   position pos = q_pos[t] of sequence b = q_seq[t]:
 *   q_idx (device) E4M3 [T, H_I, 128]: RoPE of each indexer query head
 *   w     (device) fp32 [T, H_I]: the per-head weights
 *   q     (device) bf16 bits [T, H, 576]: per head [latent query, RoPE of the RoPE query]
 *   k_idx (device) E4M3 [kv_rows, 128]: the cache row of key pos of sequence b (see
 *         dsa_batch) receives the RoPE of the indexer key
 *   kv    (device) bf16 bits [kv_rows, 576]: the same row receives [latent, RoPE of
 *         the RoPE key]; no other cache row is written
 * RoPE rotates the pairs (x[2i], x[2i+1]) of a D-dim part (D = 128 for the indexer,
 * 64 for the MLA) by the angle pos * rope_base^(-2i/D), computed in double
 * precision.  E4M3 rounds to nearest even and saturates at +-448; bf16 rounds to
 * nearest even.  A token outside its sequence (q_seq/q_pos out of range) flags
 * DSA_DEV_BAD_QUERY, one whose cache row lies outside kv_rows DSA_DEV_BAD_INDEX;
 * such tokens are not appended.
 * Workspace: dsa_workspace_size(DSA_OP_PROJECT, batch, H_I, H, 0, 0) (the fp32
 * projections and the GEMM's scratch).
 * Supported: H_I in {4, 8, ..., 64}, H in {8, 16, ..., 128}, d_model a multiple of
 * 8, every buffer 16-byte aligned.  DSA_ERR_CUDA if the GEMM library fails.
 */
dsa_status dsa_project_append(const dsa_batch *batch, const uint16_t *hidden, const uint16_t *w_all, int d_model,
                              int H_I, int H, float rope_base, uint8_t *q_idx, float *w, uint16_t *q,
                              uint8_t *k_idx, uint16_t *kv, void *ws, size_t ws_bytes, void *stream);

/*
 * Step 1, lightning indexer ("四步工作流程" 第二步 索引器評分; "两阶段流程" 1).
 *   q_idx  (device) E4M3 bytes [T, H_I, 128], row-major
 *   k_idx  (device) E4M3 bytes [total cache rows, 128]
 *   w      (device) fp32 [T, H_I] per-head weights (any scale is folded into w)
 *   scores (device) fp32 [T, ld]: scores[t*ld + s] = I[t,s] for s < n_t.
 *          Entries s >= n_t are not written.
 * Supported: H_I in {4, 8, 12, ..., 64} (multiples of 4; a count that is not a
 * power of two is padded to the next one inside the MMA, with zero weights);
 * ld >= max_kv_len, ld % 4 == 0;
 * the address of every buffer 16-byte aligned.  FP8 products are accumulated
 * in fp32 by the tensor cores; the ReLU, per-head weighting and head sum run
 * in fp32.
 */
dsa_status dsa_indexer_scores(const dsa_batch *batch, const uint8_t *q_idx, const uint8_t *k_idx,
                              const float *w, int H_I, float *scores, int64_t ld,
                              void *ws, size_t ws_bytes, void *stream);

/*
 * Step 2, top-k selection ("四步工作流程" 第三步 Top-k 選擇; "两阶段流程" 2).
 *   scores (device) fp32 [T, ld] as written by dsa_indexer_scores (only s < n_t read)
 *   idx    (device) int32 [T, k]: if n_t <= k, 0..n_t-1; otherwise the k keys with
 *          the largest score, equal scores going to the lower index (-0.0 == +0.0).
 *          Ascending index order, padded with -1 to width k.  Exact (radix select
 *          on the fp32 bit patterns); NaN scores are not supported.
 * Supported: 1 <= k <= 2048; ld >= max_kv_len, ld % 4 == 0; scores 16-byte aligned.
 */
dsa_status dsa_topk(const dsa_batch *batch, const float *scores, int64_t ld, int k, int32_t *idx,
                    void *ws, size_t ws_bytes, void *stream);

/*
 * Steps 2 -> 3 fused through a histogram ("四步工作流程" 第二步 索引器評分 feeding
 * 第三步 Top-k 選擇): the indexer's epilogue also emits, per query row, the
 * histogram of the top 11 bits of the order-preserving keys of its scores (the
 * top-k's first radix pass), and the top-k takes it instead of computing it.
 * The results are identical to dsa_indexer_scores + dsa_topk.
 *   dsa_indexer_scores_hist: as dsa_indexer_scores, plus hist (device) uint32
 *     [T, 2048] (zeroed and filled by the call).  Supported when the indexer's
 *     query groups hold at most 4 tokens of at least 32 (padded) heads: every
 *     H_I >= 36, and H_I in 20..32 with max_q_per_seq <= 4 (0: DSA_ERR_UNSUPPORTED).
 *   dsa_topk_hist: as dsa_topk, plus hist (device) as emitted for the same
 *     scores.  The clustered and the uncached top-k kernels skip their first pass
 *     over the scores; the others ignore hist.
 *   dsa_topk_uses_hist: 1 if dsa_topk_hist would use the histogram for this batch
 *     (rows long or few enough for the clustered kernel, or longer than its
 *     shared-memory cache), 0 otherwise (emitting it would then only cost time).
 */
dsa_status dsa_indexer_scores_hist(const dsa_batch *batch, const uint8_t *q_idx, const uint8_t *k_idx,
                                   const float *w, int H_I, float *scores, int64_t ld, uint32_t *hist,
                                   void *ws, size_t ws_bytes, void *stream);
dsa_status dsa_topk_hist(const dsa_batch *batch, const float *scores, int64_t ld, const uint32_t *hist, int k,
                         int32_t *idx, void *ws, size_t ws_bytes, void *stream);
int dsa_topk_uses_hist(const dsa_batch *batch, int k);

/*
 * Backward of step 3 (sparse continued training, "DeepSeek-V3.2加速技术详解" §04:
 * the model learns through the selected tokens only): gradients of the sparse MLA
 * output with respect to the queries and the latent cache rows, for an output
 * gradient d_out, with the selection held fixed (no gradient through top-k).
 * For query t, head h and selected entries i (cache rows r_i):
 *   z_i = sm_scale q.kv_i, p_i = exp(z_i - lse), D = d_out.out, dZ_i = p_i (d_out.kv_i[:512] - D)
 *   d_q[t,h]  = sm_scale sum_i dZ_i kv_i
 *   d_kv[r_i] += sm_scale dZ_i q[t,h] + p_i [d_out[t,h], 0]
 *   q, kv, idx, k, H, sm_scale: as in dsa_sparse_mla (the same call's inputs)
 *   out, lse (device) the forward's bf16 output and fp32 log-sum-exp (lse required)
 *   d_out (device) bf16 bits [T, H, 512]
 *   d_q   (device) fp32 [T, H, 576], written
 *   d_kv  (device) fp32 [kv_rows, 576]: ADDED to (atomically; a row selected by
 *         several queries or entries receives every contribution).  The caller
 *         zeroes it before the first call of a step.  Summation order varies from
 *         run to run (atomics), so d_kv is reproducible to rounding only.
 * Workspace: dsa_workspace_size(DSA_OP_MLA_BACKWARD, ...) (the status word).
 * Supported: as dsa_sparse_mla; d_q and d_kv 16-byte aligned.
 */
dsa_status dsa_sparse_mla_backward(const dsa_batch *batch, const uint16_t *q, const uint16_t *kv, const int32_t *idx,
                                   int k, int H, float sm_scale, const uint16_t *out, const float *lse,
                                   const uint16_t *d_out, float *d_q, float *d_kv, void *ws, size_t ws_bytes,
                                   void *stream);

/*
 * Step 3, sparse MLA in MQA form ("四步工作流程" 第四步 執行稀疏 MLA; "DeepSeek-V3.2
 * 加速技术详解" 3.1 MQA版MLA and 3.2 hard selection).
 *   q   (device) bf16 bits [T, H, 576] query heads (latent part then RoPE part)
 *   kv  (device) bf16 bits [total cache rows, 576]; the value of a row is its
 *       first 512 entries
 *   idx (device) int32 [T, k] local row indices; -1 entries are skipped
 *   out (device) bf16 bits [T, H, 512] = sum_i p_i * kv[row_i, :512] with
 *       p = softmax_i(sm_scale * q . kv[row_i, :576]) in fp32
 *   lse (device, may be NULL) fp32 [T, H] natural-log log-sum-exp of the scaled
 *       logits; a query with no valid index gets out = 0 and lse = -inf.
 * Supported: H in {8, 16, ..., 128} (multiples of 8, padded to 128 inside);
 * 1 <= k <= 2048.
 */
dsa_status dsa_sparse_mla(const dsa_batch *batch, const uint16_t *q, const uint16_t *kv,
                          const int32_t *idx, int k, int H, float sm_scale, uint16_t *out,
                          float *lse, void *ws, size_t ws_bytes, void *stream);

/*
 * Steps 1-3 on one stream ("四步工作流程" 第二步 to 第四步).  Scores and selected
 * indices live in `ws` (row stride: max_kv_len rounded up to 4).
 * Arguments as in the three calls above.
 */
dsa_status dsa_forward(const dsa_batch *batch, const uint8_t *q_idx, const uint8_t *k_idx,
                       const float *w, int H_I, const uint16_t *q, const uint16_t *kv, int H, int k,
                       float sm_scale, uint16_t *out, float *lse, void *ws, size_t ws_bytes,
                       void *stream);

/*
 * dsa_forward for inputs and output held in pinned host memory, with the copies
 * overlapped with the computation.  The method has no counterpart for this
 * entry point; it serves callers whose queries arrive from, and whose outputs go
 * back to, the host.  The queries are processed in chunks of
 * consecutive rows (each chunk is an independent dsa_forward over the same
 * cache, so the results are those of dsa_forward on the chunk's queries): the
 * cache and chunk c+1's queries are copied in on streams[0] while chunk c
 * computes on streams[1] and chunk c-1's output is copied out on streams[2].
 *   h_q_idx, h_w, h_q   (pinned host) query-side inputs, layouts as in dsa_forward
 *   h_k_idx, h_kv       (pinned host) the cache, batch->kv_rows rows of each
 *   q_idx, w, q, k_idx, kv (device) buffers of the same sizes, overwritten with
 *                       the copies
 *   out, lse            (device) as in dsa_forward (lse may be NULL)
 *   h_out               (pinned host) receives a copy of out
 *   streams             three streams (copy-in, compute, copy-out; they may be
 *                       the same stream, which serialises everything)
 * The call first orders itself after all work already queued on the three
 * streams that touches these buffers: copies in wait for the compute stream,
 * the computation waits for the copy-out stream.  When it returns, every copy
 * and kernel of the call has been queued and the compute stream waits for the
 * last copy out: once work queued on streams[1] after this call has
 * completed, h_out holds the output.  The host buffers must stay allocated and
 * unchanged until then (the copies read and write them asynchronously).
 * Host pointers must be page-locked (cudaHostAlloc / cudaHostRegister):
 * pageable memory returns DSA_ERR_UNSUPPORTED.
 * Workspace: dsa_workspace_size(DSA_OP_FORWARD_HOST, batch, H_I, H, k, 0) (it
 * covers the largest chunk's forward workspace).  On DSA_ERR_CUDA part of the
 * work may already be queued.
 */
dsa_status dsa_forward_host(const dsa_batch *batch, const uint8_t *h_q_idx, const float *h_w, const uint16_t *h_q,
                            const uint8_t *h_k_idx, const uint16_t *h_kv, uint8_t *q_idx, float *w, uint16_t *q,
                            uint8_t *k_idx, uint16_t *kv, int H_I, int H, int k, float sm_scale, uint16_t *out,
                            float *lse, uint16_t *h_out, void *ws, size_t ws_bytes, void *const streams[3]);

/*
 * Lightning indexer scores for callers that cannot allocate device memory.
 * The method has no counterpart for this entry point; it exists for
 * integration: some callers cannot call cudaMalloc (a host framework that
 * only hands out the tensors of the operation, a plug-in running inside
 * someone else's memory pool, code between steps that must not grow the
 * footprint), so they cannot provide the workspace `ws` that
 * dsa_indexer_scores needs for its per-call plan and status word.
 * This variant computes exactly what dsa_indexer_scores computes (same
 * arguments and results, no ws) and keeps that scratch in a fixed device array
 * inside the library instead:
 *   - Limit: num_q <= DSA_NOALLOC_MAX_Q; larger batches return
 *     DSA_ERR_UNSUPPORTED before anything is launched.  The array is about
 *     400 KB and every GPU that loads the library holds it until the process
 *     exits.
 *   - The first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *     The address is kept for the life of the process: after cudaDeviceReset
 *     (which discards the device's copy of the array) do not call this entry
 *     point again in that process.
 *   - Every call on a device shares the array and leaves its contents behind;
 *     calls whose kernels overlap on the GPU (e.g. on two streams) race on it,
 *     so serialise them.
 *   - Device-side flags (see DSA_DEV_*) land in the shared array and are not
 *     reported; host-side argument errors are.
 * Nothing is allocated: no cudaMalloc, cudaFree or allocating library call.
 */
#define DSA_NOALLOC_MAX_Q 16384
dsa_status dsa_indexer_scores_noalloc(const dsa_batch *batch, const uint8_t *q_idx, const uint8_t *k_idx,
                                      const float *w, int H_I, float *scores, int64_t ld, void *stream);

/* Pointers into a forward workspace (for inspection by tests): scores [T, ld]
 * fp32 and idx [T, k] int32.  Returns DSA_ERR_INVALID_ARGUMENT on bad input. */
dsa_status dsa_forward_ws_views(const dsa_batch *batch, int H_I, int H, int k, void *ws,
                                float **scores, int64_t *ld, int32_t **idx);

/*
 * Synchronises `stream`, copies the device status word of `ws` into *flags and
 * returns DSA_OK if it is zero, DSA_ERR_DEVICE otherwise.
 */
dsa_status dsa_read_device_status(const void *ws, uint32_t *flags, void *stream);

/*
 * Self-test of the bounded waits that guard every in-kernel spin wait, i.e. of
 * failure detection without faulting a GPU: one thread waits on a barrier that
 * nothing completes, gives up after `limit_us` microseconds (1 .. 2,000,000),
 * records DSA_DEV_TIMEOUT in the status word of `ws` (>= 256 bytes) and returns;
 * the context stays usable.  Read the flag with dsa_read_device_status.
 */
dsa_status dsa_selftest_wait_timeout(void *ws, size_t ws_bytes, uint32_t limit_us, void *stream);

/* Human-readable name of a status code (static storage). */
const char *dsa_status_string(dsa_status status);

/* DSA_ABI_VERSION of the built library. */
int dsa_abi_version(void);

/* Number of CUDA kernels the library has launched in this process so far (all
 * devices and threads; launches that failed are not counted).  Instrumentation:
 * the difference across a region counts the library's kernels in it. */
uint64_t dsa_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
