// Lightning indexer on sm_100a: I[t,s] = sum_j w[t,j] * ReLU(q_I[t,j,:] . k_I[s,:]).
//
// Page "一文讀懂DeepSeek-V3.2核心技術DSA", "DSA 的四步工作流程" step 2 (indexer
// scoring: dot products of the query against the small 128-dim key cache,
// masked, weighted by the per-head weights); page "DeepSeek 稀疏注意力路线",
// "两阶段流程" 1 (FP8, ReLU-type activation, aggregation over indexer heads).
//
// Design.  One tcgen05 GEMM per (query group, key tile):
//   A = 128 keys of one sequence (M = 128), K-major FP8 rows of 128 B;
//   B = G query tokens x H_I heads (N = G*H_I <= 256), K-major FP8 rows;
//   D = fp32 [128 keys x N] in TMEM, double buffered (2 x 256 columns).
// Keys sit in TMEM lanes, so the per-head ReLU, weighting and head sum of the
// epilogue run along one thread's own columns with no cross-lane reduction,
// and each warp stores 32 consecutive scores of a row (coalesced).
// Warp roles (576 threads): warp 0 TMA producer, warp 1 TMEM owner + MMA
// issuer, warps 2..17 epilogue (four per TMEM lane quadrant, each taking every
// fourth token of the group).  The grid is persistent (one CTA per SM); each CTA
// takes a contiguous range of work items so the resident query tile is reused
// across the key tiles of its group.  A key tile is loaded as two 64-key halves,
// each from its own cache page when the cache is paged.
#include <cstdio>

#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {

namespace {

constexpr int kEpiWarps = 16;        // four per TMEM lane quadrant, each taking every fourth token
constexpr int kIdxThreads = 64 + 32 * kEpiWarps;
constexpr int kMaxAcc = 4;           // accumulator buffers in TMEM (512 columns / N, at most 4)
constexpr int kKeyTile = 128;        // keys per item (MMA M)
constexpr int kStages = 6;           // key-tile ring depth
constexpr int kTileBytes = kKeyTile * DSA_D_INDEX;   // 16 KB
constexpr int kQBytes = 256 * DSA_D_INDEX;           // 32 KB (N <= 256)

struct __align__(8) IdxSmem {
  uint8_t q[2][kQBytes];               // 1024-aligned (offset 0): query tiles of two groups
  uint8_t k[kStages][kTileBytes];      // 1024-aligned
  float w[kEpiWarps][256];             // per epilogue warp: head weights of the group
  int32_t n_vis[kEpiWarps][64];        // per epilogue warp: visible keys per token (G <= 64)
  uint64_t k_full[kStages], k_empty[kStages];
  uint64_t q_full[2], q_empty[2];
  uint64_t acc_full[kMaxAcc], acc_empty[kMaxAcc];
  uint64_t hist_bar[4];                // per token slot: its four epilogue warps meet to flush
  uint64_t done;
  uint32_t tmem_base;
  int abort_flag;
  // last, so that a launch without histograms leaves it out of its allocation:
  uint32_t hist[4][2048];              // per token slot of a group (G <= 4): histogram of the top 11 key bits
};

// Largest g with item_off[g] <= i (item_off is non-decreasing, item_off[0] = 0).
__device__ __forceinline__ int find_group(const int32_t* item_off, int ngroups, int i) {
  int lo = 0, hi = ngroups - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (item_off[mid] <= i) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// HIST: the epilogue also emits the per-row key histograms (p.hist); a
// compile-time switch, so that the plain indexer carries none of its code.
template <int HI, bool HIST>
__global__ void __launch_bounds__(kIdxThreads, 1)
indexer_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               IndexerParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  IdxSmem& S = *reinterpret_cast<IdxSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ngroups = *p.ngroups;
  const int total = ngroups > 0 ? p.item_off[ngroups] : 0;
  const int per = (total + gridDim.x - 1) / gridDim.x;
  const int i0 = min(total, static_cast<int>(blockIdx.x) * per);
  const int i1 = min(total, i0 + per);
  const int N = p.G * HI;
  const int nacc = p.nacc;              // accumulator buffers (2 or 4), 512 / nacc columns each
  const uint32_t acc_cols = 512u / static_cast<uint32_t>(nacc);
  const int hi = p.hi;                  // real heads per token (HI = its padded column stride)
  volatile int* abort_flag = &S.abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&S.k_full[s], 1); mbar_init(&S.k_empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&S.q_full[b], 1); mbar_init(&S.q_empty[b], 1); }
    for (int a = 0; a < kMaxAcc; ++a) { mbar_init(&S.acc_full[a], 1); mbar_init(&S.acc_empty[a], 32 * kEpiWarps); }
    for (int h = 0; h < 4; ++h) mbar_init(&S.hist_bar[h], 4);
    mbar_init(&S.done, 1);
    S.abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
  }
  if (hi != HI) {
    // Tokens are loaded one by one at a stride of HI rows: the HI - hi padding
    // rows of each token stay zero (they meet zero weights in the epilogue).
    for (int i = threadIdx.x; i < 2 * kQBytes / 16; i += blockDim.x)
      reinterpret_cast<uint4*>(S.q)[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
  if (HIST)
    for (int i = threadIdx.x; i < 4 * 2048; i += blockDim.x) (&S.hist[0][0])[i] = 0u;
  if (warp == 1) tmem_alloc(&S.tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  if (i0 < i1) {
    if (warp == 0) {
      // ------------------------------------------------------------ producer
      if (lane == 0) {
        int g = find_group(p.item_off, ngroups, i0);
        int g_lo = p.item_off[g], g_hi = p.item_off[g + 1];
        int prev_g = -1, issued = 0, gq = 0;   // gq: query tiles loaded (buffer gq & 1)
        int64_t row_base = 0;                   // first cache row of the group's sequence (contiguous)
        int seq_g = 0, len_g = 0;               // the group's sequence and its length
        int st = 0;                             // key-ring stage and its phase, advanced per item
        uint32_t ph = 0;
        for (int i = i0; i < i1; ++i) {
          while (g_hi <= i) { ++g; g_lo = g_hi; g_hi = p.item_off[g + 1]; }
          const int kt = i - g_lo;
          if (g != prev_g) {
            seq_g = p.group_seq[g];
            len_g = p.kv_len[seq_g];
            row_base = p.page_size == 0 ? p.kv_offset[seq_g] : 0;
            // two query buffers: the tile of group gq reuses the buffer of group
            // gq - 2, whose MMAs must have completed; the previous group's MMAs may
            // still be running meanwhile
            const int qb = gq & 1;
            if (gq >= 2 && !mbar_wait(&S.q_empty[qb], ((gq - 2) >> 1) & 1, p.status, abort_flag)) break;
            mbar_arrive_expect_tx(&S.q_full[qb], p.G * hi * DSA_D_INDEX);
            if (hi == HI) {
              tma_load_2d(S.q[qb], &tm_q, &S.q_full[qb], 0, p.group_q0[g] * HI);
            } else {
              for (int u = 0; u < p.G; ++u)     // box = one token's hi rows
                tma_load_2d(S.q[qb] + u * HI * DSA_D_INDEX, &tm_q, &S.q_full[qb], 0, (p.group_q0[g] + u) * hi);
            }
            ++gq;
            prev_g = g;
          }
          if (!mbar_wait(&S.k_empty[st], ph ^ 1, p.status, abort_flag)) break;
          mbar_arrive_expect_tx(&S.k_full[st], kTileBytes);
          // the tile's two halves of 64 keys; with a paged cache each half lies in
          // one page (pages hold a multiple of 64 rows)
          int64_t row0 = 0;
          for (int h = 0; h < 2; ++h) {
            const int key0 = kt * kKeyTile + h * 64;
            int64_t row = row_base + key0;
            if (p.page_size != 0) {
              if (key0 < len_g) {
                const int pg = p.page_table[static_cast<int64_t>(seq_g) * p.pages_per_seq + key0 / p.page_size];
                row = static_cast<int64_t>(pg) * p.page_size + key0 % p.page_size;
                if (pg < 0 || static_cast<int64_t>(pg + 1) * p.page_size > p.kv_rows) {
                  set_status(p.status, DSA_DEV_BAD_INDEX);
                  row = 0;
                }
              } else {
                row = row0;                     // keys past the sequence end are masked
              }
            }
            if (h == 0) row0 = row;
            tma_load_2d(S.k[st] + h * 64 * DSA_D_INDEX, &tm_k, &S.k_full[st], 0, static_cast<int>(row));
          }
          ++issued;
          if (++st == kStages) { st = 0; ph ^= 1; }
        }
        // Never leave with a copy in flight: wait (bounded) for the last load of each stage.
        for (int n = max(0, issued - kStages); n < issued; ++n)
          mbar_wait(&S.k_full[n % kStages], (n / kStages) & 1, p.status, nullptr);
        for (int gl = max(0, gq - 2); gl < gq; ++gl) mbar_wait(&S.q_full[gl & 1], (gl >> 1) & 1, p.status, nullptr);
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        const uint32_t idesc = instr_desc(0, 0, false, false, kKeyTile, N);
        int g = find_group(p.item_off, ngroups, i0);
        int g_hi = p.item_off[g + 1];
        int prev_g = -1, gm = 0;                // gm: groups started (query buffer (gm - 1) & 1)
        // Issue must stay lean (this thread shares its scheduler with epilogue
        // warps): descriptors are built once and stepped by adds to the 14-bit
        // start-address field (16-byte units); stages advance by counters.
        const uint64_t kdesc0 = smem_desc_sw128(smem_u32(S.k[0]), 16, 1024);
        const uint64_t qdesc0 = smem_desc_sw128(smem_u32(S.q[0]), 16, 1024);
        uint64_t qd = qdesc0, kd = kdesc0;
        uint32_t d = tmem;
        int st = 0, a = 0;
        uint32_t ph = 0, aph = 0;
        for (int i = i0; i < i1; ++i) {
          while (g_hi <= i) { ++g; g_hi = p.item_off[g + 1]; }
          if (g != prev_g) {
            if (!mbar_wait(&S.q_full[gm & 1], (gm >> 1) & 1, p.status, abort_flag)) break;
            qd = qdesc0 + static_cast<uint64_t>((gm & 1) * (kQBytes / 16));
            ++gm;
            prev_g = g;
          }
          if (!mbar_wait(&S.acc_empty[a], aph ^ 1, p.status, abort_flag)) break;
          tc_fence_after();
          if (!mbar_wait(&S.k_full[st], ph, p.status, abort_flag)) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < DSA_D_INDEX / 32; ++kk)
            umma_f8(d, kd + static_cast<uint64_t>(kk * 2), qd + static_cast<uint64_t>(kk * 2), idesc, kk > 0 ? 1u : 0u);
          umma_commit(&S.k_empty[st]);
          umma_commit(&S.acc_full[a]);
          const bool last_of_group = (i + 1 == i1) || (g_hi <= i + 1);
          if (last_of_group) umma_commit(&S.q_empty[(gm - 1) & 1]);
          if (++st == kStages) { st = 0; ph ^= 1; kd = kdesc0; } else { kd += kTileBytes / 16; }
          if (++a == nacc) { a = 0; aph ^= 1; d = tmem; } else { d += acc_cols; }
        }
        umma_commit(&S.done);
        mbar_wait(&S.done, 0, p.status, nullptr);
      }
    } else {
      // ------------------------------------------------------------ epilogue
      // Warp-uniform control flow: lane 0 waits on barriers, the warp follows.
      const int ew = warp - 2;                    // 0..15
      const int quad = warp & 3;                  // TMEM lane quadrant of this warp
      const int tsub = ew >> 2;                   // tokens tsub, tsub + 4, ... of each group
      const int row = quad * 32 + lane;           // key within the tile
      float* sw = S.w[ew];
      int32_t* snv = S.n_vis[ew];
      int g = find_group(p.item_off, ngroups, i0);
      int g_lo = p.item_off[g], g_hi = p.item_off[g + 1];
      int prev_g = -1, cnt = 0, q0 = 0;
      int a = 0;                                  // accumulator buffer and its phase, advanced per item
      uint32_t aph = 0;
      // Histogram emission (p.hist set; groups of at most 4 tokens, so token slot =
      // tsub): the four warps of a token slot count the top 11 key bits of the
      // group's scores in shared memory; when the group ends they meet, each adds
      // a quarter of the bins to the row's global histogram, and meet again.
      uint32_t nh = 0;                            // completed phases of hist_bar[tsub]
      auto hsync = [&]() -> bool {
        __syncwarp();
        int ok = 1;
        if (lane == 0) {
          mbar_arrive(&S.hist_bar[tsub]);
          ok = mbar_wait(&S.hist_bar[tsub], nh & 1, p.status, abort_flag) ? 1 : 0;
        }
        ++nh;
        return __shfl_sync(0xffffffffu, ok, 0) != 0;
      };
      auto flush = [&](int fq0, int fcnt) -> bool {
        if (!hsync()) return false;
        if (tsub < fcnt) {
          uint32_t* hs = S.hist[tsub];
          uint32_t* hg = p.hist + static_cast<int64_t>(fq0 + tsub) * 2048;
          for (int b = quad * 512 + lane; b < quad * 512 + 512; b += 32) {
            const uint32_t v = hs[b];
            if (v) {
              atomicAdd(hg + b, v);
              hs[b] = 0u;
            }
          }
        }
        return hsync();
      };
      bool hist_ok = true;
      for (int i = i0; i < i1; ++i) {
        while (g_hi <= i) { ++g; g_lo = g_hi; g_hi = p.item_off[g + 1]; }
        const int kt = i - g_lo;
        if (g != prev_g) {
          if (HIST && prev_g >= 0 && !(hist_ok = flush(q0, cnt))) break;
          __syncwarp();
          q0 = p.group_q0[g];
          cnt = p.group_cnt[g];
          // all loads of the group's weights and visible counts in flight at once
          constexpr int kWPer = 256 / 32;         // G * HI <= 256
          float wv[kWPer];
          int nv[2];
#pragma unroll
          for (int u = 0; u < kWPer; ++u) {
            const int j = lane + 32 * u, tok = j / HI, h = j - tok * HI;
            wv[u] = (j < cnt * HI && h < hi) ? __ldg(p.w + static_cast<int64_t>(q0 + tok) * hi + h) : 0.f;
          }
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int j = lane + 32 * u;
            nv[u] = j < cnt ? __ldg(p.q_nvis + q0 + j) : 0;
          }
#pragma unroll
          for (int u = 0; u < kWPer; ++u) sw[lane + 32 * u] = wv[u];
#pragma unroll
          for (int u = 0; u < 2; ++u) snv[lane + 32 * u] = max(0, nv[u]);   // cnt <= 64
          __syncwarp();
          prev_g = g;
        }
        int ok = 1;
        if (lane == 0) ok = mbar_wait(&S.acc_full[a], aph, p.status, abort_flag) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        tc_fence_after();
        const int s = kt * kKeyTile + row;
        const uint32_t tbase = tmem + (static_cast<uint32_t>(quad * 32) << 16) + a * acc_cols;
        if constexpr (HI >= 32) {
          // one token per pass: its HI head columns, ReLU, then the weighted head
          // sum in packed pairs (fma.rn.f32x2) over four independent accumulators
          for (int tok = tsub; tok < cnt; tok += 4) {
            const float* wr = &sw[tok * HI];
            float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                             make_float2(0.f, 0.f)};
#pragma unroll
            for (int c = 0; c < HI / 32; ++c) {      // 32 head columns per TMEM load
              uint32_t v[32];
              tmem_ld32(tbase + tok * HI + c * 32, v);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 32; j += 8) {
                const float4 wa = *reinterpret_cast<const float4*>(wr + c * 32 + j);
                const float4 wb = *reinterpret_cast<const float4*>(wr + c * 32 + j + 4);
                const int u = (j >> 3) & 1;
                acc[2 * u] = ffma2(make_float2(wa.x, wa.y),
                                   make_float2(fmaxf(__uint_as_float(v[j + 0]), 0.f), fmaxf(__uint_as_float(v[j + 1]), 0.f)),
                                   acc[2 * u]);
                acc[2 * u + 1] = ffma2(make_float2(wa.z, wa.w),
                                       make_float2(fmaxf(__uint_as_float(v[j + 2]), 0.f), fmaxf(__uint_as_float(v[j + 3]), 0.f)),
                                       acc[2 * u + 1]);
                acc[2 * u] = ffma2(make_float2(wb.x, wb.y),
                                   make_float2(fmaxf(__uint_as_float(v[j + 4]), 0.f), fmaxf(__uint_as_float(v[j + 5]), 0.f)),
                                   acc[2 * u]);
                acc[2 * u + 1] = ffma2(make_float2(wb.z, wb.w),
                                       make_float2(fmaxf(__uint_as_float(v[j + 6]), 0.f), fmaxf(__uint_as_float(v[j + 7]), 0.f)),
                                       acc[2 * u + 1]);
              }
            }
            const float sum = ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) +
                              ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
            const bool vis = s < snv[tok];
            if (vis) p.scores[static_cast<int64_t>(q0 + tok) * p.ld + s] = sum;
            if constexpr (HIST) {
              // warp-aggregated: lanes whose bins agree with the first lane's add once
              const uint32_t bin = order_key(sum) >> 21;
              const uint32_t inmask = __ballot_sync(0xffffffffu, vis);
              if (inmask) {
                const int leader = __ffs(inmask) - 1;
                const uint32_t b0 = __shfl_sync(0xffffffffu, bin, leader);
                const uint32_t same = __ballot_sync(0xffffffffu, vis && bin == b0);
                if (lane == leader) atomicAdd(&S.hist[tsub][b0], static_cast<uint32_t>(__popc(same)));
                if (vis && bin != b0) atomicAdd(&S.hist[tsub][bin], 1u);
              }
            }
          }
        } else {
          constexpr int TPC = 32 / HI;             // tokens per 32-column chunk
          const int nchunks = (cnt * HI + 31) / 32;
          for (int c = tsub; c < nchunks; c += 4) {
            uint32_t v[32];
            tmem_ld32(tbase + c * 32, v);
            tmem_ld_wait();
            float acc[TPC];
#pragma unroll
            for (int u = 0; u < TPC; ++u) acc[u] = 0.f;
            const float* wr = &sw[c * 32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              acc[j / HI] = fmaf(wr[j], fmaxf(__uint_as_float(v[j]), 0.f), acc[j / HI]);
            }
#pragma unroll
            for (int u = 0; u < TPC; ++u) {
              const int tok = c * TPC + u;
              if (tok < cnt && s < snv[tok]) p.scores[static_cast<int64_t>(q0 + tok) * p.ld + s] = acc[u];
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&S.acc_empty[a]);
        if (++a == nacc) { a = 0; aph ^= 1; }
      }
      if (HIST && hist_ok && prev_g >= 0 && !*abort_flag) flush(q0, cnt);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ----------------------------------------------------------------- planning
// One CTA.  Forms groups of at most G consecutive queries of one sequence,
// records each group's first query, size and sequence, the number of 128-key
// tiles its last query needs, and the exclusive prefix of those counts.
constexpr int kPlanThreads = 1024;

__device__ int block_inclusive_scan(int v, int* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += x;
  }
  if (lane == 31) scratch[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int t = lane < (blockDim.x >> 5) ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += x;
    }
    scratch[lane] = t;
  }
  __syncthreads();
  if (warp > 0) v += scratch[warp - 1];
  __syncthreads();
  return v;
}

// Visible keys of query t (q_pos + 1), or -1 when its sequence or position is
// out of range (the query then gets no scores).
__device__ __forceinline__ int visible_keys(const IndexerParams& p, int t, int B, int64_t kv_rows) {
  const int seq = p.q_seq[t];
  if (seq < 0 || seq >= B) return -1;
  const int len = p.kv_len[seq];
  const int pos = p.q_pos[t];
  if (len < 0 || len > p.max_kv_len || pos < 0 || pos >= len) return -1;
  if (p.page_size == 0) {
    const int64_t off = p.kv_offset[seq];
    if (off < 0 || off + len > kv_rows) return -1;
  } else if (len > static_cast<int64_t>(p.pages_per_seq) * p.page_size) {
    return -1;
  }
  return pos + 1;
}

__global__ void __launch_bounds__(kPlanThreads) indexer_plan_kernel(IndexerParams p, int T, int B, int64_t kv_rows) {
  __shared__ int scratch[32];
  __shared__ int carry_groups, carry_run_start, carry_tiles;
  if (threadIdx.x == 0) { carry_groups = 0; carry_run_start = 0; carry_tiles = 0; }
  __syncthreads();
  // Pass 1: leaders and group records.
  for (int base = 0; base < T; base += kPlanThreads) {
    const int t = base + threadIdx.x;
    int seq = -1;
    bool run_start = false;
    if (t < T) {
      seq = p.q_seq[t];
      run_start = (t == 0) || (p.q_seq[t - 1] != seq);
      const int nv = visible_keys(p, t, B, kv_rows);
      p.q_nvis[t] = nv;
      if (nv < 0) set_status(p.status, DSA_DEV_BAD_QUERY);
    }
    // last run start at or before t: inclusive max-scan of (run_start ? t : -1)
    int rs = run_start ? t : -1;
    {
      const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, rs, o);
        if (lane >= o) rs = max(rs, x);
      }
      if (lane == 31) scratch[warp] = rs;
      __syncthreads();
      if (warp == 0) {
        int m = scratch[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int x = __shfl_up_sync(0xffffffffu, m, o);
          if (lane >= o) m = max(m, x);
        }
        scratch[lane] = m;
      }
      __syncthreads();
      if (warp > 0) rs = max(rs, scratch[warp - 1]);
      rs = max(rs, carry_run_start);
      __syncthreads();
    }
    const bool leader = (t < T) && (((t - rs) % p.G) == 0);
    const int inc = block_inclusive_scan(leader ? 1 : 0, scratch);
    if (leader) {
      const int gi = carry_groups + inc - 1;
      int cnt = 1, maxn = 0;
      for (int u = 0; u < p.G && t + u < T; ++u) {
        const int tu = t + u;
        if (u > 0 && p.q_seq[tu] != seq) break;
        cnt = u + 1;
        maxn = max(maxn, max(0, visible_keys(p, tu, B, kv_rows)));
      }
      p.group_q0[gi] = t;
      p.group_cnt[gi] = cnt;
      p.group_seq[gi] = (seq >= 0 && seq < B) ? seq : 0;
      p.group_tiles[gi] = (maxn + kKeyTile - 1) / kKeyTile;
    }
    __syncthreads();
    if (threadIdx.x == kPlanThreads - 1) {
      carry_groups += inc;
      carry_run_start = max(carry_run_start, rs);
    }
    __syncthreads();
  }
  const int ngroups = carry_groups;
  // Pass 2: exclusive prefix of tile counts.
  for (int base = 0; base < ngroups; base += kPlanThreads) {
    const int gi = base + threadIdx.x;
    const int v = gi < ngroups ? p.group_tiles[gi] : 0;
    const int inc = block_inclusive_scan(v, scratch);
    if (gi < ngroups) p.item_off[gi] = carry_tiles + inc - v;
    __syncthreads();
    if (threadIdx.x == kPlanThreads - 1) carry_tiles += inc;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    p.item_off[ngroups] = carry_tiles;
    *p.ngroups = ngroups;
  }
}

}  // namespace

static_assert(sizeof(IdxSmem) + 1024 <= 232448, "indexer shared memory exceeds the 227 KB per-CTA limit");
size_t indexer_smem_bytes() { return sizeof(IdxSmem) + 1024; }
// without histograms the trailing histogram array is not allocated
static size_t indexer_smem_bytes_for(bool hist) {
  return hist ? indexer_smem_bytes() : indexer_smem_bytes() - sizeof(uint32_t) * 4 * 2048;
}

// hi_pad: the token column stride (a power of two, 4..64); p.hi <= hi_pad is H_I.
cudaError_t launch_indexer(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const IndexerParams& p, int hi_pad,
                           int T, int B, int64_t kv_rows, int num_sms, cudaStream_t stream) {
  indexer_plan_kernel<<<1, kPlanThreads, 0, stream>>>(p, T, B, kv_rows);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  count_launches(1);
  const size_t smem = indexer_smem_bytes_for(p.hist != nullptr);
  auto launch = [&](auto kern) -> cudaError_t {
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    kern<<<num_sms, kIdxThreads, smem, stream>>>(tm_q, tm_k, p);
    err = cudaGetLastError();
    if (err == cudaSuccess) count_launches(1);
    return err;
  };
  if (p.hist) {                        // the host allows histograms only with >= 32 padded heads
    switch (hi_pad) {
      case 32: return launch(indexer_kernel<32, true>);
      case 64: return launch(indexer_kernel<64, true>);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (hi_pad) {
    case 4: return launch(indexer_kernel<4, false>);
    case 8: return launch(indexer_kernel<8, false>);
    case 16: return launch(indexer_kernel<16, false>);
    case 32: return launch(indexer_kernel<32, false>);
    case 64: return launch(indexer_kernel<64, false>);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dsa
