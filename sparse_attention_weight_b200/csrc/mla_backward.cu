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
// Design (CUDA cores, fp32).  One CTA (256 threads) per (query, chunk of HC =
// 32/16/8 heads): the chunk's queries and output gradients stay in shared memory
// as fp32, the selected rows stream through in tiles of 32 (gathered by index,
// converted to fp32); a tile without a usable entry is skipped.  Per tile, three
// register-tiled products:
//   1. z and dO.v for every (head, row): each thread a 4-head x 4-row tile over a
//      1/KS slice of the 576 (512) dims, float4 loads, even and odd dims summed
//      in the two lanes of packed fma.rn.f32x2 pairs, the KS slices summed by
//      shuffles; then p and dZ, one row per slice lane.
//   2. dQ += dZ . rows: each thread HC/8 heads x 18 dims, accumulated in
//      registers over all tiles (written once, no atomics), dim pairs with one
//      packed fma.rn.f32x2.
//   3. each row's d_kv contribution summed over the chunk's heads: each thread 4
//      rows x 18 dims, added to the fp32 gradient cache with float2 atomics (a
//      row selected by several queries collects all their contributions).
// Row strides in shared memory are padded by 4 floats (16-byte aligned rows
// whose banks shift by 4 from one row to the next).
#include <cuda_bf16.h>

#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {

namespace {

constexpr int kBwdThreads = 256;
constexpr int kRT = 32;                  // selected rows per tile
constexpr int kQS = DSA_D_QK + 4;        // padded fp32 stride of a 576-wide row
constexpr int kOS = DSA_D_V + 4;         // padded fp32 stride of a 512-wide row
constexpr int kDPer = DSA_D_QK / 32;     // 18 dims per lane in products 2 and 3 (float2 pairs lane*2 + 64j)

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
  const int lane = tid & 31, warp = tid >> 5;
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

  // product 1 mapping: tile (hb, rb) of 4 heads x 4 rows, KS lanes per tile
  constexpr int KS = 128 / HC;                     // 4, 8, 16
  const int tile = tid / KS, ks = tid % KS;
  const int hb = tile / (kRT / 4), rb = tile % (kRT / 4);
  // product 2 mapping: heads warp*HPW .. +HPW-1, dims lane*2 + 64j
  constexpr int HPW = HC / 8;                      // 4, 2, 1
  float dq[HPW][kDPer];
#pragma unroll
  for (int a = 0; a < HPW; ++a)
#pragma unroll
    for (int j = 0; j < kDPer; ++j) dq[a][j] = 0.f;
  const float scale = p.sm_scale;

  const int32_t* idx_row = p.idx + static_cast<int64_t>(t) * p.k;
  for (int e0 = 0; rows_ok && e0 < p.k; e0 += kRT) {
    // cache rows of the tile's entries
    bool any = false;
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
      any = r >= 0;
    }
    if (!__syncthreads_or(any)) continue;          // no usable entry in this tile
    // gather the rows (8 bf16 per 16-byte load), zeros for unused entries
    for (int i = tid; i < kRT * (DSA_D_QK / 8); i += kBwdThreads) {
      const int r = i / (DSA_D_QK / 8), c8 = i - r * (DSA_D_QK / 8);
      const int64_t row = S.row_of[r];
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (row >= 0) v = __ldg(reinterpret_cast<const uint4*>(p.kv + row * DSA_D_QK) + c8);
      float4* dst = reinterpret_cast<float4*>(&S.rows[r][c8 * 8]);
      dst[0] = make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                           __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
      dst[1] = make_float4(__uint_as_float(v.z << 16), __uint_as_float(v.z & 0xffff0000u),
                           __uint_as_float(v.w << 16), __uint_as_float(v.w & 0xffff0000u));
    }
    __syncthreads();

    // ---- product 1: z and dO.v of heads 4hb.., rows 4rb.., dim chunks ks, ks+KS, ...
    {
      // z and dO.v accumulate even and odd dims in the two lanes of a packed pair
      float2 z2[4][4], dp2[4][4];
      float z[4][4], dp[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) { z2[a][b] = make_float2(0.f, 0.f); dp2[a][b] = make_float2(0.f, 0.f); }
#pragma unroll 2
      for (int c = ks; c < DSA_D_QK / 4; c += KS) {
        const int d = c * 4;
        float4 qa[4], ra[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) qa[a] = *reinterpret_cast<const float4*>(&S.q[hb * 4 + a][d]);
#pragma unroll
        for (int b = 0; b < 4; ++b) ra[b] = *reinterpret_cast<const float4*>(&S.rows[rb * 4 + b][d]);
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            z2[a][b] = ffma2(make_float2(qa[a].x, qa[a].y), make_float2(ra[b].x, ra[b].y), z2[a][b]);
            z2[a][b] = ffma2(make_float2(qa[a].z, qa[a].w), make_float2(ra[b].z, ra[b].w), z2[a][b]);
          }
        if (d < DSA_D_V) {
#pragma unroll
          for (int a = 0; a < 4; ++a) {
            const float4 oa = *reinterpret_cast<const float4*>(&S.dout[hb * 4 + a][d]);
#pragma unroll
            for (int b = 0; b < 4; ++b) {
              dp2[a][b] = ffma2(make_float2(oa.x, oa.y), make_float2(ra[b].x, ra[b].y), dp2[a][b]);
              dp2[a][b] = ffma2(make_float2(oa.z, oa.w), make_float2(ra[b].z, ra[b].w), dp2[a][b]);
            }
          }
        }
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          z[a][b] = z2[a][b].x + z2[a][b].y;
          dp[a][b] = dp2[a][b].x + dp2[a][b].y;
        }
      // sum the KS slices (lanes tile*KS .. +KS-1 of one warp)
#pragma unroll
      for (int o = KS / 2; o > 0; o >>= 1)
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            z[a][b] += __shfl_xor_sync(0xffffffffu, z[a][b], o);
            dp[a][b] += __shfl_xor_sync(0xffffffffu, dp[a][b], o);
          }
      // p and dZ: slice lane ks < 4 takes row 4rb + ks
      if (ks < 4) {
        const int r = rb * 4 + ks;
        const bool row_used = S.row_of[r] >= 0;
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          const int h = hb * 4 + a;
          float zz = z[a][0], dd = dp[a][0];
#pragma unroll
          for (int b = 1; b < 4; ++b)
            if (ks == b) { zz = z[a][b]; dd = dp[a][b]; }
          const bool used = row_used && S.lse[h] != -INFINITY;
          const float pv = used ? __expf(scale * zz - S.lse[h]) : 0.f;
          S.p[h][r] = pv;
          S.dz[h][r] = pv * (dd - S.dh[h]);
        }
      }
    }
    __syncthreads();

    // ---- product 2: dQ += dZ . rows (heads warp*HPW.., dims lane*2 + 64j)
#pragma unroll 2
    for (int r = 0; r < kRT; ++r) {
      float g[HPW];
#pragma unroll
      for (int a = 0; a < HPW; ++a) g[a] = S.dz[warp * HPW + a][r];
#pragma unroll
      for (int j = 0; j < kDPer / 2; ++j) {
        const float2 v = *reinterpret_cast<const float2*>(&S.rows[r][lane * 2 + 64 * j]);
#pragma unroll
        for (int a = 0; a < HPW; ++a) {
          const float2 r2 = ffma2(make_float2(g[a], g[a]), v, make_float2(dq[a][2 * j], dq[a][2 * j + 1]));
          dq[a][2 * j] = r2.x;
          dq[a][2 * j + 1] = r2.y;
        }
      }
    }

    // ---- product 3: the d_kv contributions of rows 4*warp.. (dims lane*2 + 64j)
    {
      float acc[4][kDPer];
#pragma unroll
      for (int b = 0; b < 4; ++b)
#pragma unroll
        for (int j = 0; j < kDPer; ++j) acc[b][j] = 0.f;
#pragma unroll 1
      for (int h = 0; h < HC; ++h) {
        float g[4], pv[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          g[b] = scale * S.dz[h][warp * 4 + b];
          pv[b] = S.p[h][warp * 4 + b];
        }
#pragma unroll
        for (int j = 0; j < kDPer / 2; ++j) {
          const float2 qv = *reinterpret_cast<const float2*>(&S.q[h][lane * 2 + 64 * j]);
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const float2 r2 = ffma2(make_float2(g[b], g[b]), qv, make_float2(acc[b][2 * j], acc[b][2 * j + 1]));
            acc[b][2 * j] = r2.x;
            acc[b][2 * j + 1] = r2.y;
          }
          if (64 * j < DSA_D_V) {                  // dims 64j + lane*2 < 512 for j < 8
            const float2 ov = *reinterpret_cast<const float2*>(&S.dout[h][lane * 2 + 64 * j]);
#pragma unroll
            for (int b = 0; b < 4; ++b) {
              const float2 r2 = ffma2(make_float2(pv[b], pv[b]), ov, make_float2(acc[b][2 * j], acc[b][2 * j + 1]));
              acc[b][2 * j] = r2.x;
              acc[b][2 * j + 1] = r2.y;
            }
          }
        }
      }
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int64_t row = S.row_of[warp * 4 + b];
        if (row < 0) continue;
        float* dst = p.d_kv + row * DSA_D_QK + lane * 2;       // 8-byte aligned
#pragma unroll
        for (int j = 0; j < kDPer / 2; ++j)
          atomicAdd(reinterpret_cast<float2*>(dst + 64 * j), make_float2(acc[b][2 * j], acc[b][2 * j + 1]));
      }
    }
    __syncthreads();                               // rows, p, dz and row_of are rewritten by the next tile
  }
#pragma unroll
  for (int a = 0; a < HPW; ++a) {
    float* dqo = p.d_q + (static_cast<int64_t>(t) * H + h0 + warp * HPW + a) * DSA_D_QK + lane * 2;
#pragma unroll
    for (int j = 0; j < kDPer / 2; ++j)
      *reinterpret_cast<float2*>(dqo + 64 * j) = make_float2(scale * dq[a][2 * j], scale * dq[a][2 * j + 1]);
  }
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
