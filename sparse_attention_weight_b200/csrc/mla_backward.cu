// Backward pass of the sparse MLA on sm_100a (training through the sparse
// attention with the selection held fixed).
//
// Page "DeepSeek-V3.2加速技术详解" §04 (sparse continued training: the model learns
// through the selected tokens only); page "一文讀懂DeepSeek-V3.2核心技術DSA" (DSA
// keeps the model trainable end to end).  For query t, head h, selected entries i
// (rows r_i of the latent cache, value = the first 512 entries of the row):
//   z_i = s q.kv_i, p_i = exp(z_i - lse), D = dO.o, dZ_i = p_i (dO.v_i - D)
//   dQ = s sum_i dZ_i kv_i,   dKV[r_i] += s dZ_i q + p_i [dO, 0]
// with o and lse the forward's output and log-sum-exp.
//
// Design (a first, CUDA-core path).  One CTA per (query, chunk of HC heads):
// the chunk's queries and output gradients stay in shared memory as fp32, the
// selected rows stream through in tiles of 16 (gathered by index, converted to
// fp32); per tile the CTA forms z, p, dZ for the chunk's heads, adds into dQ
// (registers) and forms each row's dKV contribution summed over the chunk's
// heads, which it adds to the fp32 gradient cache with vector atomics (a row
// selected by several queries collects all their contributions).  Rows are
// padded to an odd stride in shared memory so that threads reading different
// rows at the same column hit different banks.
#include <cuda_bf16.h>

#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {

namespace {

constexpr int kBwdThreads = 256;
constexpr int kRT = 16;                  // selected rows per tile
constexpr int kQS = DSA_D_QK + 1;        // padded fp32 stride of a 576-wide row
constexpr int kOS = DSA_D_V + 1;         // padded fp32 stride of a 512-wide row

template <int HC>
struct BwdSmem {
  float q[HC][kQS];
  float dout[HC][kOS];
  float rows[kRT][kQS];
  float p[HC][kRT];
  float dz[HC][kRT];
  float dh[HC];
  float lse[HC];
  int64_t row_of[kRT];                   // cache row of each tile entry, -1 if unused
};

__device__ __forceinline__ float bf16f(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

template <int HC>
__global__ void __launch_bounds__(kBwdThreads, 1) mla_backward_kernel(MlaBwdParams p) {
  extern __shared__ __align__(16) uint8_t bwd_raw[];
  BwdSmem<HC>& S = *reinterpret_cast<BwdSmem<HC>*>(bwd_raw);
  const int t = blockIdx.x;
  const int h0 = blockIdx.y * HC;
  const int tid = threadIdx.x;
  const int H = p.H;
  // sequence of the query
  const int seq = p.q_seq[t];
  const bool seq_ok = seq >= 0 && seq < p.num_seqs;
  const int len = seq_ok ? p.kv_len[seq] : 0;
  const int64_t base = seq_ok && p.page_size == 0 ? p.kv_offset[seq] : 0;
  const bool rows_ok = seq_ok && len >= 0 &&
                       (p.page_size == 0 ? base >= 0 && base + len <= p.kv_rows
                                         : len <= static_cast<int64_t>(p.pages_per_seq) * p.page_size);
  if (!rows_ok && tid == 0 && blockIdx.y == 0) set_status(p.status, DSA_DEV_BAD_QUERY);

  // queries, output gradients (fp32), lse and D = dO . o of the chunk's heads
  for (int i = tid; i < HC * DSA_D_QK; i += kBwdThreads) {
    const int h = i / DSA_D_QK, d = i - h * DSA_D_QK;
    S.q[h][d] = bf16f(p.q[(static_cast<int64_t>(t) * H + h0 + h) * DSA_D_QK + d]);
  }
  for (int i = tid; i < HC * DSA_D_V; i += kBwdThreads) {
    const int h = i / DSA_D_V, d = i - h * DSA_D_V;
    S.dout[h][d] = bf16f(p.d_out[(static_cast<int64_t>(t) * H + h0 + h) * DSA_D_V + d]);
  }
  {
    // D per head: 256 / HC threads per head, each a slice of the 512 dims
    constexpr int TPH = kBwdThreads / HC;
    const int h = tid / TPH, part = tid % TPH;
    float acc = 0.f;
    const int64_t orow = (static_cast<int64_t>(t) * H + h0 + h) * DSA_D_V;
    for (int d = part; d < DSA_D_V; d += TPH)
      acc = fmaf(bf16f(p.d_out[orow + d]), bf16f(p.out[orow + d]), acc);
#pragma unroll
    for (int o = TPH / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (part == 0) {
      S.dh[h] = acc;
      S.lse[h] = p.lse[static_cast<int64_t>(t) * H + h0 + h];
    }
  }
  __syncthreads();

  // dQ accumulators: thread = (head hq, 576 / (256 / HC) consecutive dims)
  constexpr int QTPH = kBwdThreads / HC;           // threads per head for dQ
  constexpr int QPER = DSA_D_QK / QTPH;            // dims per thread
  const int hq = tid / QTPH, dq0 = (tid % QTPH) * QPER;
  float dq[QPER];
#pragma unroll
  for (int j = 0; j < QPER; ++j) dq[j] = 0.f;
  // dKV contributions: thread = (tile row rk, 36 consecutive dims)
  constexpr int KTPR = kBwdThreads / kRT;          // 16 threads per row
  constexpr int KPER = DSA_D_QK / KTPR;            // 36 dims per thread
  const int rk = tid / KTPR, dk0 = (tid % KTPR) * KPER;
  const float scale = p.sm_scale;

  const int32_t* idx_row = p.idx + static_cast<int64_t>(t) * p.k;
  for (int e0 = 0; rows_ok && e0 < p.k; e0 += kRT) {
    // cache rows of the tile's entries
    if (tid < kRT) {
      const int e = e0 + tid;
      const int v = e < p.k ? idx_row[e] : -1;
      int64_t r = -1;
      if (v >= len) set_status(p.status, DSA_DEV_BAD_INDEX);
      if (v >= 0 && v < len) {
        if (p.page_size == 0) {
          r = base + v;
        } else {
          const int pg = p.page_table[static_cast<int64_t>(seq) * p.pages_per_seq + v / p.page_size];
          r = static_cast<int64_t>(pg) * p.page_size + v % p.page_size;
          if (pg < 0 || r >= p.kv_rows) {
            set_status(p.status, DSA_DEV_BAD_INDEX);
            r = -1;
          }
        }
      }
      S.row_of[tid] = r;
    }
    __syncthreads();
    // gather the rows (8 bf16 per 16-byte load), zeros for unused entries
    for (int i = tid; i < kRT * (DSA_D_QK / 8); i += kBwdThreads) {
      const int r = i / (DSA_D_QK / 8), c8 = i - r * (DSA_D_QK / 8);
      const int64_t row = S.row_of[r];
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (row >= 0) v = __ldg(reinterpret_cast<const uint4*>(p.kv + row * DSA_D_QK) + c8);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      float* dst = &S.rows[r][c8 * 8];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        dst[2 * u] = __uint_as_float(w[u] << 16);
        dst[2 * u + 1] = __uint_as_float(w[u] & 0xffff0000u);
      }
    }
    __syncthreads();
    // z, p, dZ for every (head, entry) pair of the tile
    for (int pr = tid; pr < HC * kRT; pr += kBwdThreads) {
      const int h = pr / kRT, r = pr - h * kRT;
      float z = 0.f, dp = 0.f;
      for (int d = 0; d < DSA_D_V; ++d) {
        const float kvd = S.rows[r][d];
        z = fmaf(S.q[h][d], kvd, z);
        dp = fmaf(S.dout[h][d], kvd, dp);
      }
      for (int d = DSA_D_V; d < DSA_D_QK; ++d) z = fmaf(S.q[h][d], S.rows[r][d], z);
      const bool used = S.row_of[r] >= 0 && S.lse[h] != -INFINITY;
      const float pv = used ? __expf(scale * z - S.lse[h]) : 0.f;
      S.p[h][r] = pv;
      S.dz[h][r] = pv * (dp - S.dh[h]);
    }
    __syncthreads();
    // dQ += dZ . rows
#pragma unroll 1
    for (int r = 0; r < kRT; ++r) {
      const float g = S.dz[hq][r];
      const float* src = &S.rows[r][dq0];
#pragma unroll
      for (int j = 0; j < QPER; ++j) dq[j] = fmaf(g, src[j], dq[j]);
    }
    // this row's dKV contribution over the chunk's heads, added to the cache gradient
    const int64_t row = S.row_of[rk];
    if (row >= 0) {
      float acc[KPER];
#pragma unroll
      for (int j = 0; j < KPER; ++j) acc[j] = 0.f;
#pragma unroll 1
      for (int h = 0; h < HC; ++h) {
        const float g = scale * S.dz[h][rk];
        const float pv = S.p[h][rk];
        const float* qs = &S.q[h][dk0];
        const float* os = &S.dout[h][dk0];
#pragma unroll
        for (int j = 0; j < KPER; ++j) {
          acc[j] = fmaf(g, qs[j], acc[j]);
          if (dk0 + j < DSA_D_V) acc[j] = fmaf(pv, os[j], acc[j]);
        }
      }
      float* dst = p.d_kv + row * DSA_D_QK + dk0;      // dk0 = 36 * lane-of-row: 16-byte aligned
#pragma unroll
      for (int j = 0; j < KPER; j += 4)
        atomicAdd(reinterpret_cast<float4*>(dst + j), make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]));
    }
    __syncthreads();
  }
  float* dqo = p.d_q + (static_cast<int64_t>(t) * H + h0 + hq) * DSA_D_QK + dq0;
#pragma unroll
  for (int j = 0; j < QPER; ++j) dqo[j] = scale * dq[j];
}

template <int HC>
cudaError_t launch_hc(const MlaBwdParams& p, cudaStream_t stream) {
  const size_t smem = sizeof(BwdSmem<HC>);
  cudaError_t e = cudaFuncSetAttribute(mla_backward_kernel<HC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  mla_backward_kernel<HC><<<dim3(p.T, p.H / HC), kBwdThreads, smem, stream>>>(p);
  e = cudaGetLastError();
  if (e == cudaSuccess) count_launches(1);
  return e;
}

}  // namespace

cudaError_t launch_mla_backward(const MlaBwdParams& p, cudaStream_t stream) {
  if (p.T == 0) return cudaSuccess;
  if (p.H % 32 == 0) return launch_hc<32>(p, stream);
  if (p.H % 16 == 0) return launch_hc<16>(p, stream);
  return launch_hc<8>(p, stream);
}

}  // namespace dsa
