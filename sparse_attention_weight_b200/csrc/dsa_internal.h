// Kernel parameter blocks and launchers shared between the kernels and the C ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace dsa {

struct IndexerParams {
  const float* w;            // [T, H_I]
  float* scores;             // [T, ld]
  int64_t ld;
  const int32_t* q_seq;      // [T]
  const int32_t* q_pos;      // [T]
  const int64_t* kv_offset;  // [B] (contiguous layout)
  const int32_t* kv_len;     // [B]
  const int32_t* page_table; // [B, pages_per_seq] (paged layout, page_size > 0)
  int page_size;             // 0 = contiguous rows from kv_offset
  int pages_per_seq;
  int64_t kv_rows;           // rows of the k_idx buffer
  uint32_t* hist;            // [T, 2048] histogram of the top 11 key bits per row (zeroed), or null
  // plan (workspace)
  int32_t* group_q0;         // [T]
  int32_t* group_cnt;        // [T]
  int32_t* group_seq;        // [T]
  int32_t* group_tiles;      // [T]
  int32_t* item_off;         // [T + 1]
  int32_t* ngroups;          // [1]
  int32_t* q_nvis;           // [T] visible keys per query, -1 = invalid query
  uint32_t* status;
  int G;                     // query tokens per group (N = G * padded H_I)
  int hi;                    // H_I, heads per query token (a multiple of 4, <= 64)
  int nacc;                  // accumulator buffers in TMEM: 4 when N <= 128, else 2
  int max_kv_len;
};

struct TopkParams {
  const float* scores;       // [T, ld]
  const uint32_t* hist;      // [T, 2048] per-row histogram of the top 11 key bits, or null
  int64_t ld;
  int32_t* idx;              // [T, k]
  int k;
  const int32_t* q_seq;
  const int32_t* q_pos;
  const int32_t* kv_len;
  int num_seqs;
  int max_kv_len;
  uint32_t* status;
};

struct MlaParams {
  const uint16_t* q;         // [T, H, 576] bf16
  const uint16_t* kv;        // [rows, 576] bf16
  const int32_t* idx;        // [T, k]
  int k;
  int H;
  float sm_scale_log2;       // sm_scale * log2(e)
  float sm_scale;
  uint16_t* out;             // [T, H, 512] bf16
  float* lse;                // [T, H] or null
  const int32_t* q_seq;
  const int32_t* q_pos;
  const int64_t* kv_offset;  // contiguous layout
  const int32_t* kv_len;
  const int32_t* page_table; // [B, pages_per_seq] (paged layout, page_size > 0)
  int page_size;             // 0 = contiguous rows from kv_offset
  int pages_per_seq;
  int num_seqs;
  int64_t kv_rows;
  int T;
  int splits;                // index-list splits per query (1 = no combine pass)
  float* part_o;             // [T, splits, H, 512] fp32 (splits > 1)
  float* part_lse;           // [T, splits, H]       fp32 (splits > 1)
  uint32_t* status;
};

struct ProjParams {
  float* y;                  // [T, n_all] fp32 projections (workspace)
  uint8_t* q_idx;            // [T, H_I, 128] E4M3
  float* w;                  // [T, H_I]
  uint16_t* q;               // [T, H, 576] bf16
  uint8_t* k_cache;          // [kv_rows, 128] E4M3
  uint16_t* kv_cache;        // [kv_rows, 576] bf16
  const int32_t* q_seq;
  const int32_t* q_pos;
  const int64_t* kv_offset;  // contiguous layout
  const int32_t* kv_len;
  const int32_t* page_table; // paged layout (page_size > 0)
  int page_size;
  int pages_per_seq;
  int num_seqs;
  int64_t kv_rows;
  int T;
  int n_all;                 // rows of the stacked projection matrix
  int hi;                    // H_I
  int heads;                 // H
  float rope_base;
  uint32_t* status;
};

struct MlaBwdParams {
  const uint16_t* q;         // [T, H, 576] bf16
  const uint16_t* kv;        // [rows, 576] bf16
  const int32_t* idx;        // [T, k]
  int k;
  int H;
  float sm_scale;
  const uint16_t* out;       // [T, H, 512] bf16, the forward's output
  const float* lse;          // [T, H], the forward's log-sum-exp
  const uint16_t* d_out;     // [T, H, 512] bf16
  float* d_q;                // [T, H, 576]
  float* d_kv;               // [rows, 576], accumulated
  const int32_t* q_seq;
  const int64_t* kv_offset;
  const int32_t* kv_len;
  const int32_t* page_table;
  int page_size;
  int pages_per_seq;
  int num_seqs;
  int64_t kv_rows;
  int T;
  uint32_t* status;
};
cudaError_t launch_mla_backward(const MlaBwdParams& p, cudaStream_t stream);

// Counts kernel launches made by the library (dsa_launch_count).
void count_launches(int n);

size_t project_gemm_workspace_bytes();
cudaError_t launch_project(const ProjParams& p, const uint16_t* hidden, const uint16_t* w_all, int d_model,
                           void* gemm_ws, size_t gemm_ws_bytes, cudaStream_t stream, bool* gemm_failed);
size_t indexer_smem_bytes();
size_t mla_smem_bytes();
cudaError_t launch_indexer(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const IndexerParams& p, int hi_pad,
                           int T, int B, int64_t kv_rows, int num_sms, cudaStream_t stream);
cudaError_t launch_topk(const TopkParams& p, int T, cudaStream_t stream);
// Whether the top-k kernel chosen for these rows takes an emitted histogram as
// its first radix pass (the clustered and the uncached streaming kernels).
bool topk_uses_hist(int max_kv_len, int T, int sms);
cudaError_t launch_sparse_mla(const MlaParams& p, const CUtensorMap& tm_q, cudaStream_t stream);

}  // namespace dsa
