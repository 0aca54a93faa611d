// The step before the DSA path on sm_100a: projections of the new tokens' hidden
// states, rotary position embedding, FP8 / bf16 storage casts and cache append.
//
// Page "一文讀懂DeepSeek-V3.2核心技術DSA", "DSA 的四步工作流程" step 1 (queries and
// keys projected from the hidden states with rotary embeddings folded in, plus
// per-head weights projected from the hidden state); page "DeepSeek 稀疏注意力路线",
// V3's MLA (the token's hidden state is down-projected to the cached latent;
// position enters through a separate, decoupled RoPE channel); page
// "DeepSeek-V3.2加速技术详解" 3.1 (MQA form: the query lives in the latent space).
//
// Design.  One plain GEMM, Y = h W^T over the stacked weight matrix (bf16 x bf16
// -> fp32, cuBLASLt), then one kernel per token row of Y that rotates the RoPE
// parts, casts every part to its storage format and writes the query-side
// outputs and the token's two cache rows.  The epilogue is HBM-bound (it reads
// 4 B and writes 1-2 B per projected value): one CTA per token, the rotation
// angles computed once per CTA in double precision (pos reaches 2^17, so an
// fp32 angle pos * freq would be off by up to ~1e-2 rad), the pairs rotated in
// fp32, vectorised loads and stores.
#include <cublasLt.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <mutex>

#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {

namespace {

constexpr int kProjThreads = 256;

__device__ __forceinline__ uint32_t bf16x2(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// E4M3, round to nearest even, saturating to +-448 (the storage format of the
// indexer's queries and keys).
__device__ __forceinline__ uint16_t e4m3x2(float a, float b) {
  return static_cast<uint16_t>(__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}

__global__ void __launch_bounds__(kProjThreads) project_epilogue_kernel(ProjParams p) {
  __shared__ float cs128[64][2];   // cos, sin of the 64 pair angles of a 128-dim head
  __shared__ float cs64[32][2];    // ... of a 64-dim RoPE part
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  const int seq = p.q_seq[t];
  const int pos = p.q_pos[t];
  const bool q_ok = seq >= 0 && seq < p.num_seqs && pos >= 0 && pos < p.kv_len[seq];
  // cache row of the new token (-1: not appended)
  int64_t row = -1;
  if (q_ok) {
    if (p.page_size == 0) {
      const int64_t off = p.kv_offset[seq];
      row = (off >= 0 && off + pos < p.kv_rows) ? off + pos : -1;
    } else {
      const int pg = p.page_table[static_cast<int64_t>(seq) * p.pages_per_seq + pos / p.page_size];
      const int64_t r = static_cast<int64_t>(pg) * p.page_size + pos % p.page_size;
      row = (pg >= 0 && r < p.kv_rows) ? r : -1;
    }
  }
  if (tid == 0 && row < 0) set_status(p.status, q_ok ? DSA_DEV_BAD_INDEX : DSA_DEV_BAD_QUERY);
  if (tid < 96) {
    const int D = tid < 64 ? 128 : 64;
    const int i = tid < 64 ? tid : tid - 64;
    const double ang = static_cast<double>(q_ok ? pos : 0) * exp(-2.0 * i / D * log(static_cast<double>(p.rope_base)));
    double s, c;
    sincos(ang, &s, &c);
    float* dst = tid < 64 ? cs128[i] : cs64[i];
    dst[0] = static_cast<float>(c);
    dst[1] = static_cast<float>(s);
  }
  __syncthreads();
  const float* y = p.y + static_cast<int64_t>(t) * p.n_all;
  const int HI = p.hi, H = p.heads;
  // offsets of the stacked projection (rows of W = columns of Y)
  const int o_qi = 0, o_ki = o_qi + HI * DSA_D_INDEX, o_w = o_ki + DSA_D_INDEX, o_lat = o_w + HI;
  const int o_kr = o_lat + 512, o_ql = o_kr + 64, o_qr = o_ql + H * 512;

  // indexer query heads and key: rotate each pair, cast to E4M3 (4 values per thread step)
  for (int j = tid; j < (HI + 1) * 32; j += kProjThreads) {
    const int head = j >> 5;                      // head HI is the key
    const int quad = j & 31;                      // values 4*quad .. +3 of the 128
    const float4 v = *reinterpret_cast<const float4*>(y + (head < HI ? o_qi + head * 128 : o_ki) + quad * 4);
    const float* c0 = cs128[quad * 2];
    const float* c1 = cs128[quad * 2 + 1];
    const float a0 = v.x * c0[0] - v.y * c0[1], b0 = v.x * c0[1] + v.y * c0[0];
    const float a1 = v.z * c1[0] - v.w * c1[1], b1 = v.z * c1[1] + v.w * c1[0];
    const uint32_t packed = static_cast<uint32_t>(e4m3x2(a0, b0)) | (static_cast<uint32_t>(e4m3x2(a1, b1)) << 16);
    if (head < HI) {
      *reinterpret_cast<uint32_t*>(p.q_idx + (static_cast<int64_t>(t) * HI + head) * DSA_D_INDEX + quad * 4) = packed;
    } else if (row >= 0) {
      *reinterpret_cast<uint32_t*>(p.k_cache + row * DSA_D_INDEX + quad * 4) = packed;
    }
  }
  // per-head weights (fp32)
  for (int j = tid; j < HI; j += kProjThreads) p.w[static_cast<int64_t>(t) * HI + j] = y[o_w + j];
  // latent row [latent 512, rotated RoPE key 64] -> bf16 cache row (4 values per step)
  if (row >= 0) {
    uint16_t* kvr = p.kv_cache + row * DSA_D_QK;
    for (int j = tid; j < DSA_D_QK / 4; j += kProjThreads) {
      const float4 v = *reinterpret_cast<const float4*>(y + o_lat + j * 4);   // o_kr = o_lat + 512
      float a0 = v.x, b0 = v.y, a1 = v.z, b1 = v.w;
      if (j >= 128) {
        const int i = (j - 128) * 2;             // pair index within the 64-dim RoPE part
        a0 = v.x * cs64[i][0] - v.y * cs64[i][1];
        b0 = v.x * cs64[i][1] + v.y * cs64[i][0];
        a1 = v.z * cs64[i + 1][0] - v.w * cs64[i + 1][1];
        b1 = v.z * cs64[i + 1][1] + v.w * cs64[i + 1][0];
      }
      *reinterpret_cast<uint2*>(kvr + j * 4) = make_uint2(bf16x2(a0, b0), bf16x2(a1, b1));
    }
  }
  // MLA query heads: [latent query 512, rotated RoPE query 64] -> bf16 (4 values per step)
  uint16_t* qrow = p.q + static_cast<int64_t>(t) * H * DSA_D_QK;
  for (int j = tid; j < H * (DSA_D_QK / 4); j += kProjThreads) {
    const int head = j / (DSA_D_QK / 4);
    const int c4 = j - head * (DSA_D_QK / 4);    // 4-value group of the 576
    float4 v;
    if (c4 < 128) {
      v = *reinterpret_cast<const float4*>(y + o_ql + head * 512 + c4 * 4);
    } else {
      const int i = (c4 - 128) * 2;
      const float4 r = *reinterpret_cast<const float4*>(y + o_qr + head * 64 + (c4 - 128) * 4);
      v.x = r.x * cs64[i][0] - r.y * cs64[i][1];
      v.y = r.x * cs64[i][1] + r.y * cs64[i][0];
      v.z = r.z * cs64[i + 1][0] - r.w * cs64[i + 1][1];
      v.w = r.z * cs64[i + 1][1] + r.w * cs64[i + 1][0];
    }
    *reinterpret_cast<uint2*>(qrow + head * DSA_D_QK + c4 * 4) = make_uint2(bf16x2(v.x, v.y), bf16x2(v.z, v.w));
  }
}

// One cuBLASLt handle per device, created on first use.
cublasLtHandle_t lt_handle() {
  static std::mutex mu;
  static cublasLtHandle_t handles[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!handles[dev] && cublasLtCreate(&handles[dev]) != CUBLAS_STATUS_SUCCESS) handles[dev] = nullptr;
  return handles[dev];
}

}  // namespace

size_t project_gemm_workspace_bytes() { return 32u << 20; }

cudaError_t launch_project(const ProjParams& p, const uint16_t* hidden, const uint16_t* w_all, int d_model,
                           void* gemm_ws, size_t gemm_ws_bytes, cudaStream_t stream, bool* gemm_failed) {
  *gemm_failed = false;
  if (p.T == 0) return cudaSuccess;
  // Y [T, N] (row-major) = h [T, d] W[N, d]^T, i.e. in column-major terms
  // Y' [N, T] = W'^T [N, d] X' [d, T] with W' = W viewed as [d, N], X' = h as [d, T].
  cublasLtHandle_t h = lt_handle();
  cublasLtMatmulDesc_t op = nullptr;
  cublasLtMatrixLayout_t la = nullptr, lb = nullptr, lc = nullptr;
  cublasLtMatmulPreference_t pref = nullptr;
  bool ok = h != nullptr;
  ok = ok && cublasLtMatmulDescCreate(&op, CUBLAS_COMPUTE_32F, CUDA_R_32F) == CUBLAS_STATUS_SUCCESS;
  const cublasOperation_t ta = CUBLAS_OP_T, tb = CUBLAS_OP_N;
  ok = ok && cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSA, &ta, sizeof(ta)) == CUBLAS_STATUS_SUCCESS;
  ok = ok && cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSB, &tb, sizeof(tb)) == CUBLAS_STATUS_SUCCESS;
  ok = ok && cublasLtMatrixLayoutCreate(&la, CUDA_R_16BF, d_model, p.n_all, d_model) == CUBLAS_STATUS_SUCCESS;
  ok = ok && cublasLtMatrixLayoutCreate(&lb, CUDA_R_16BF, d_model, p.T, d_model) == CUBLAS_STATUS_SUCCESS;
  ok = ok && cublasLtMatrixLayoutCreate(&lc, CUDA_R_32F, p.n_all, p.T, p.n_all) == CUBLAS_STATUS_SUCCESS;
  ok = ok && cublasLtMatmulPreferenceCreate(&pref) == CUBLAS_STATUS_SUCCESS;
  ok = ok && cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &gemm_ws_bytes,
                                                  sizeof(gemm_ws_bytes)) == CUBLAS_STATUS_SUCCESS;
  cublasLtMatmulHeuristicResult_t heur = {};
  int found = 0;
  ok = ok && cublasLtMatmulAlgoGetHeuristic(h, op, la, lb, lc, lc, pref, 1, &heur, &found) == CUBLAS_STATUS_SUCCESS &&
       found > 0;
  const float alpha = 1.f, beta = 0.f;
  ok = ok && cublasLtMatmul(h, op, &alpha, w_all, la, hidden, lb, &beta, p.y, lc, p.y, lc, &heur.algo, gemm_ws,
                            gemm_ws_bytes, stream) == CUBLAS_STATUS_SUCCESS;
  if (pref) cublasLtMatmulPreferenceDestroy(pref);
  if (lc) cublasLtMatrixLayoutDestroy(lc);
  if (lb) cublasLtMatrixLayoutDestroy(lb);
  if (la) cublasLtMatrixLayoutDestroy(la);
  if (op) cublasLtMatmulDescDestroy(op);
  if (!ok) {
    *gemm_failed = true;
    return cudaErrorUnknown;
  }
  count_launches(1);
  project_epilogue_kernel<<<p.T, kProjThreads, 0, stream>>>(p);
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) count_launches(1);
  return e;
}

}  // namespace dsa
