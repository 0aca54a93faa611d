// Fine-grained top-k selection on sm_100a.
//
// Page "一文讀懂DeepSeek-V3.2核心技術DSA", "DSA 的四步工作流程" step 3: keep the
// 2048 highest-scoring tokens of the context per query, all of them when the
// context holds <= k tokens; page "DeepSeek-V3.2加速技术详解" 3.2: the rest are
// dropped.  Equal scores go to the lower index; -0.0 equals +0.0; output in
// ascending index order, padded with -1.
//
// Design.  One CTA per query row.  Scores map to order-preserving 32-bit keys;
// the k-th largest key is found exactly by three histogram passes over 11, 11
// and 10 key bits (2048-bin shared-memory histograms, warp-aggregated with
// match.any so hot bins take one atomic per warp), then one output pass emits,
// in index order, every key above the threshold and the first `need` keys equal
// to it.  The output pass needs a single block scan per 2048 elements: with
// gt/eq counts before an element, its slot is gt_before + min(eq_before, need).
// Rows up to the shared-memory cache size are read from HBM once; longer rows
// are re-read from L2 by each pass.  Loads are float4 (16 B per thread,
// 512 B per warp, coalesced).
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {

namespace {

constexpr int kThreads = 512;
constexpr int kPer = 4;
constexpr int kStep = kThreads * kPer;   // elements per block step
constexpr int kCacheMax = 32768;         // keys cached in shared memory at most (128 KB)

__device__ __forceinline__ uint32_t order_key(float x) {
  uint32_t b = __float_as_uint(x);
  if ((b & 0x7fffffffu) == 0) b = 0;     // -0.0 == +0.0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

struct Ctx {
  const float* row;
  uint32_t* cache;     // null when the row is not cached
  int n;
};

// Keys of elements i..i+3 (invalid entries get `valid` cleared).
__device__ __forceinline__ void load_keys(const Ctx& c, int i, bool from_cache, bool fill_cache,
                                          uint32_t (&k)[kPer], bool (&valid)[kPer]) {
  if (from_cache) {
    const uint4 v = *reinterpret_cast<const uint4*>(c.cache + i);
    k[0] = v.x; k[1] = v.y; k[2] = v.z; k[3] = v.w;
#pragma unroll
    for (int u = 0; u < kPer; ++u) valid[u] = (i + u) < c.n;
    return;
  }
  if (i + kPer <= c.n) {
    const float4 f = __ldg(reinterpret_cast<const float4*>(c.row + i));
    k[0] = order_key(f.x); k[1] = order_key(f.y); k[2] = order_key(f.z); k[3] = order_key(f.w);
#pragma unroll
    for (int u = 0; u < kPer; ++u) valid[u] = true;
  } else {
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      valid[u] = (i + u) < c.n;
      k[u] = valid[u] ? order_key(__ldg(c.row + i + u)) : 0u;
    }
  }
  if (fill_cache && i < c.n) {
    *reinterpret_cast<uint4*>(c.cache + i) = make_uint4(k[0], k[1], k[2], k[3]);
  }
}

// Inclusive block scan over kThreads ints; *total receives the block sum.
__device__ __forceinline__ uint32_t block_scan(uint32_t v, uint32_t* scratch, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t x = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += x;
  }
  if (lane == 31) scratch[warp] = v;
  __syncthreads();
  if (warp == 0) {
    uint32_t t = lane < kThreads / 32 ? scratch[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t x = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += x;
    }
    scratch[lane] = t;
  }
  __syncthreads();
  if (warp > 0) v += scratch[warp - 1];
  *total = scratch[kThreads / 32 - 1];
  __syncthreads();
  return v;
}

// Histogram of key bits [shift, shift+bits) over keys whose bits above `fshift`
// equal `prefix` (fshift = 32: no filter).
__device__ void hist_pass(const Ctx& c, bool from_cache, bool fill_cache, uint32_t* hist, int shift, int bits,
                          int fshift, uint32_t prefix) {
  const int lane = threadIdx.x & 31;
  const uint32_t mask = (1u << bits) - 1u;
  for (int base = 0; base < c.n; base += kStep) {
    const int i = base + threadIdx.x * kPer;
    uint32_t k[kPer];
    bool valid[kPer];
    load_keys(c, i, from_cache, fill_cache, k, valid);
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const bool in = valid[u] && (fshift >= 32 || (k[u] >> fshift) == prefix);
      const uint32_t bin = in ? ((k[u] >> shift) & mask) : 0xffffffffu;
      const uint32_t peers = __match_any_sync(0xffffffffu, bin);
      if (in && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], static_cast<uint32_t>(__popc(peers)));
    }
  }
}

// Finds the bin holding the kneed-th largest key, counting from the top bin,
// and how many keys of that bin are still needed.
__device__ void find_bin(const uint32_t* hist, int nbins, uint32_t kneed, uint32_t* scratch, uint32_t* out_bin,
                         uint32_t* out_rem) {
  const int per = nbins / kThreads;
  const int b0 = threadIdx.x * per;
  uint32_t local = 0;
  for (int b = 0; b < per; ++b) local += hist[b0 + b];
  uint32_t total;
  const uint32_t incl = block_scan(local, scratch, &total);
  uint32_t above = total - incl;          // keys in bins owned by higher threads
  for (int b = per - 1; b >= 0; --b) {
    const uint32_t h = hist[b0 + b];
    if (above < kneed && above + h >= kneed) {
      *out_bin = static_cast<uint32_t>(b0 + b);
      *out_rem = kneed - above;
    }
    above += h;
  }
  __syncthreads();
}

// n of query row t (visible keys), or -1 for an invalid query; rows with n <= k
// (and invalid ones) are written here and the function returns -1 / 0 for them.
__device__ __forceinline__ int row_length(const TopkParams& p, int t, int32_t* out) {
  const int k = p.k;
  int n = -1;
  const int seq = p.q_seq[t];
  if (seq >= 0 && seq < p.num_seqs) {
    const int len = p.kv_len[seq];
    const int pos = p.q_pos[t];
    if (len >= 0 && len <= p.max_kv_len && pos >= 0 && pos < len) n = pos + 1;
  }
  if (n < 0) {
    if (threadIdx.x == 0) set_status(p.status, DSA_DEV_BAD_QUERY);
    for (int j = threadIdx.x; j < k; j += kThreads) out[j] = -1;
    return -1;
  }
  if (n <= k) {
    for (int j = threadIdx.x; j < k; j += kThreads) out[j] = j < n ? j : -1;
    return 0;
  }
  return n;
}

// Exact top-k of row c (n > k) by three histogram passes (11, 11, 10 key bits)
// and one output pass over the row: from the shared-memory cache when c.cache
// is set (the first pass fills it), from L2 otherwise.
__device__ void select_streaming(const Ctx& c, int k, int32_t* out, uint32_t* hist, uint32_t* scratch,
                                 uint32_t* sel) {
  const bool cached = c.cache != nullptr;
  const int n = c.n;
  // pass 1: bits 31..21
  for (int b = threadIdx.x; b < 2048; b += kThreads) hist[b] = 0;
  __syncthreads();
  hist_pass(c, false, cached, hist, 21, 11, 32, 0);
  __syncthreads();
  find_bin(hist, 2048, static_cast<uint32_t>(k), scratch, &sel[0], &sel[1]);
  const uint32_t b1 = sel[0], r1 = sel[1];
  __syncthreads();

  // pass 2: bits 20..10 among keys with the pass-1 prefix
  for (int b = threadIdx.x; b < 2048; b += kThreads) hist[b] = 0;
  __syncthreads();
  hist_pass(c, cached, false, hist, 10, 11, 21, b1);
  __syncthreads();
  find_bin(hist, 2048, r1, scratch, &sel[0], &sel[1]);
  const uint32_t b2 = sel[0], r2 = sel[1];
  __syncthreads();

  // pass 3: bits 9..0
  const uint32_t pre2 = (b1 << 11) | b2;
  for (int b = threadIdx.x; b < 1024; b += kThreads) hist[b] = 0;
  __syncthreads();
  hist_pass(c, cached, false, hist, 0, 10, 10, pre2);
  __syncthreads();
  find_bin(hist, 1024, r2, scratch, &sel[0], &sel[1]);
  const uint32_t tau = (pre2 << 10) | sel[0];
  const uint32_t need = sel[1];             // keys equal to tau to take, lowest indices first
  __syncthreads();

  // output pass, index order
  uint32_t gt_base = 0, eq_base = 0;
  for (int base = 0; base < n; base += kStep) {
    const int i = base + threadIdx.x * kPer;
    uint32_t kk[kPer];
    bool valid[kPer];
    load_keys(c, i, cached, false, kk, valid);
    uint32_t cgt = 0, ceq = 0;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      cgt += (valid[u] && kk[u] > tau) ? 1u : 0u;
      ceq += (valid[u] && kk[u] == tau) ? 1u : 0u;
    }
    const uint32_t packed = cgt | (ceq << 16);
    uint32_t total;
    const uint32_t incl = block_scan(packed, scratch, &total);
    const uint32_t excl = incl - packed;
    uint32_t gt_before = gt_base + (excl & 0xffffu);
    uint32_t eq_before = eq_base + (excl >> 16);
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      if (!valid[u]) continue;
      if (kk[u] > tau) {
        const uint32_t slot = gt_before + min(eq_before, need);
        if (slot < static_cast<uint32_t>(k)) out[slot] = i + u;
        ++gt_before;
      } else if (kk[u] == tau) {
        const uint32_t slot = gt_before + eq_before;
        if (eq_before < need && slot < static_cast<uint32_t>(k)) out[slot] = i + u;
        ++eq_before;
      }
    }
    gt_base += total & 0xffffu;
    eq_base += total >> 16;
  }
}

__global__ void __launch_bounds__(kThreads) topk_kernel(TopkParams p, int cache_elems) {
  extern __shared__ __align__(16) uint32_t tk_smem[];
  uint32_t* hist = tk_smem;                 // 2048
  uint32_t* scratch = hist + 2048;          // 32
  uint32_t* sel = scratch + 32;             // [0] bin, [1] remaining
  uint32_t* cache = sel + 32;               // cache_elems (16-byte aligned: offset 2112 words)
  const int t = blockIdx.x;
  int32_t* out = p.idx + static_cast<int64_t>(t) * p.k;
  const int n = row_length(p, t, out);
  if (n <= 0) return;
  const Ctx c{p.scores + static_cast<int64_t>(t) * p.ld, n <= cache_elems ? cache : nullptr, n};
  select_streaming(c, p.k, out, hist, scratch, sel);
}

// ---------------------------------------------------------------- long rows
// Rows too long for the shared-memory cache.  Pass 1 histograms the top 13 key
// bits over the row; pass 2 reads the row again and compacts, in index order,
// every key whose top bits reach the selected bin (all keys above it are taken,
// the bin's keys are candidates) into a shared-memory list.  The remaining 19
// bits are resolved on the list (10 + 9 bits) and the output pass runs over the
// list, so the row is read twice instead of four times.  A row whose list would
// overflow (a bin holding more than kListCap - k keys, e.g. massive ties) falls
// back to the streaming passes.  Used when the rows are few (see launch_topk).
constexpr int kHiBits = 13;
constexpr int kHiShift = 32 - kHiBits;    // 19
constexpr int kListCap = 8192;

// Histogram of bits [shift, shift+bits) over list keys whose bits above `fshift` equal `prefix`.
__device__ void hist_list(const uint32_t* keys, int m, uint32_t* hist, int shift, int bits, int fshift,
                          uint32_t prefix) {
  const int lane = threadIdx.x & 31;
  const uint32_t mask = (1u << bits) - 1u;
  for (int base = 0; base < m; base += kThreads) {
    const int i = base + threadIdx.x;
    const bool in = i < m && (keys[i < m ? i : 0] >> fshift) == prefix;
    const uint32_t bin = in ? ((keys[i] >> shift) & mask) : 0xffffffffu;
    const uint32_t peers = __match_any_sync(0xffffffffu, bin);
    if (in && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], static_cast<uint32_t>(__popc(peers)));
  }
}

__global__ void __launch_bounds__(kThreads) topk_long_kernel(TopkParams p) {
  extern __shared__ __align__(16) uint32_t tk_smem[];
  uint32_t* hist = tk_smem;                           // 1 << kHiBits
  uint32_t* scratch = hist + (1 << kHiBits);          // 32
  uint32_t* sel = scratch + 32;                       // [0] bin, [1] remaining
  uint32_t* lkey = sel + 32;                          // kListCap
  int32_t* lidx = reinterpret_cast<int32_t*>(lkey + kListCap);   // kListCap
  const int t = blockIdx.x;
  const int k = p.k;
  int32_t* out = p.idx + static_cast<int64_t>(t) * k;
  const int n = row_length(p, t, out);
  if (n <= 0) return;
  const Ctx c{p.scores + static_cast<int64_t>(t) * p.ld, nullptr, n};

  // pass 1: top 13 bits over the row
  for (int b = threadIdx.x; b < (1 << kHiBits); b += kThreads) hist[b] = 0;
  __syncthreads();
  hist_pass(c, false, false, hist, kHiShift, kHiBits, 32, 0);
  __syncthreads();
  find_bin(hist, 1 << kHiBits, static_cast<uint32_t>(k), scratch, &sel[0], &sel[1]);
  const uint32_t b1 = sel[0], r1 = sel[1];
  const uint32_t m_total = (static_cast<uint32_t>(k) - r1) + hist[b1];   // keys at or above bin b1
  __syncthreads();
  if (m_total > static_cast<uint32_t>(kListCap)) {    // block-uniform: fall back to streaming
    select_streaming(c, k, out, hist, scratch, sel);
    return;
  }

  // pass 2: compact keys with top bits >= b1, in index order
  uint32_t m = 0;
  for (int base = 0; base < n; base += kStep) {
    const int i = base + threadIdx.x * kPer;
    uint32_t kk[kPer];
    bool valid[kPer];
    load_keys(c, i, false, false, kk, valid);
    uint32_t cnt = 0;
#pragma unroll
    for (int u = 0; u < kPer; ++u) cnt += (valid[u] && (kk[u] >> kHiShift) >= b1) ? 1u : 0u;
    uint32_t total;
    const uint32_t incl = block_scan(cnt, scratch, &total);
    uint32_t pos = m + incl - cnt;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      if (valid[u] && (kk[u] >> kHiShift) >= b1) {
        if (pos < static_cast<uint32_t>(kListCap)) {
          lkey[pos] = kk[u];
          lidx[pos] = i + u;
        }
        ++pos;
      }
    }
    m += total;
  }
  __syncthreads();
  const int mi = static_cast<int>(min(m, static_cast<uint32_t>(kListCap)));

  // passes 3 and 4 on the list: bits 18..9, then 8..0
  for (int b = threadIdx.x; b < 1024; b += kThreads) hist[b] = 0;
  __syncthreads();
  hist_list(lkey, mi, hist, 9, 10, kHiShift, b1);
  __syncthreads();
  find_bin(hist, 1024, r1, scratch, &sel[0], &sel[1]);
  const uint32_t b2 = sel[0], r2 = sel[1];
  __syncthreads();
  const uint32_t pre2 = (b1 << 10) | b2;
  for (int b = threadIdx.x; b < 512; b += kThreads) hist[b] = 0;
  __syncthreads();
  hist_list(lkey, mi, hist, 0, 9, 9, pre2);
  __syncthreads();
  find_bin(hist, 512, r2, scratch, &sel[0], &sel[1]);
  const uint32_t tau = (pre2 << 9) | sel[0];
  const uint32_t need = sel[1];             // keys equal to tau to take, lowest indices first
  __syncthreads();

  // output pass over the list (index order)
  uint32_t gt_base = 0, eq_base = 0;
  for (int base = 0; base < mi; base += kStep) {
    const int i = base + threadIdx.x * kPer;
    uint32_t kk[kPer];
    bool valid[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      valid[u] = i + u < mi;
      kk[u] = valid[u] ? lkey[i + u] : 0u;
    }
    uint32_t cgt = 0, ceq = 0;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      cgt += (valid[u] && kk[u] > tau) ? 1u : 0u;
      ceq += (valid[u] && kk[u] == tau) ? 1u : 0u;
    }
    const uint32_t packed = cgt | (ceq << 16);
    uint32_t total;
    const uint32_t incl = block_scan(packed, scratch, &total);
    const uint32_t excl = incl - packed;
    uint32_t gt_before = gt_base + (excl & 0xffffu);
    uint32_t eq_before = eq_base + (excl >> 16);
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      if (!valid[u]) continue;
      if (kk[u] > tau) {
        const uint32_t slot = gt_before + min(eq_before, need);
        if (slot < static_cast<uint32_t>(k)) out[slot] = lidx[i + u];
        ++gt_before;
      } else if (kk[u] == tau) {
        const uint32_t slot = gt_before + eq_before;
        if (eq_before < need && slot < static_cast<uint32_t>(k)) out[slot] = lidx[i + u];
        ++eq_before;
      }
    }
    gt_base += total & 0xffffu;
    eq_base += total >> 16;
  }
}

}  // namespace

cudaError_t launch_topk(const TopkParams& p, int T, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  int cache_elems = ((p.max_kv_len + kStep - 1) / kStep) * kStep;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess)
    sms = 148;
  // Long rows.  With few rows (at most two per SM: decode) each CTA has an SM to
  // itself and reading the row twice instead of four times wins; with many rows
  // the streaming kernel, four CTAs per SM, keeps more loads in flight.
  if (cache_elems > kCacheMax && T <= 2 * sms) {      // two reads and a candidate list
    const size_t smem = ((1 << kHiBits) + 64 + 2 * kListCap) * sizeof(uint32_t);
    cudaError_t e = cudaFuncSetAttribute(topk_long_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    topk_long_kernel<<<T, kThreads, smem, stream>>>(p);
    e = cudaGetLastError();
    if (e == cudaSuccess) count_launches(1);
    return e;
  }
  if (cache_elems > kCacheMax) cache_elems = 0;       // long rows stream from L2
  const size_t smem = (2048 + 64) * sizeof(uint32_t) + static_cast<size_t>(cache_elems) * sizeof(uint32_t);
  cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  topk_kernel<<<T, kThreads, smem, stream>>>(p, cache_elems);
  e = cudaGetLastError();
  if (e == cudaSuccess) count_launches(1);
  return e;
}

}  // namespace dsa
