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
// and 10 key bits (2048-bin shared-memory histograms; a warp whose keys share
// one bin makes one atomic, found with ballots), then one output pass emits,
// in index order, every key above the threshold and the first `need` keys equal
// to it.  The output pass needs a single block scan per 2048 elements: with
// gt/eq counts before an element, its slot is gt_before + min(eq_before, need).
// Rows up to the shared-memory cache size are read from HBM once; longer rows
// are re-read from L2 by each pass.  Loads are float4 (16 B per thread,
// 512 B per warp, coalesced).  A cached row of at least 5k keys whose keys at
// or above the first pass's bin fit a list (and are at most a quarter of the
// row) is compacted, in index order, into that list of positions, and the two
// later passes and the output run over the list instead of the whole row.
#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {

namespace {

constexpr int kThreads = 512;
constexpr int kPer = 4;
constexpr int kStep = kThreads * kPer;   // elements per block step
constexpr int kCacheMax = 32768;         // keys cached in shared memory at most (128 KB)
constexpr int kClusterMinLen = 8192;     // rows at least this long may share a cluster of CTAs
constexpr int kClusterSegMax = 20480;    // keys cached per CTA of a cluster (80 KB: two CTAs per SM)
// Cached rows: positions of the keys at or above the pass-1 threshold bin, in
// index order (about k plus one bin), so that the later passes and the output
// run over this list instead of the whole cached row.  The host sizes the list
// within the shared memory left over at the kernel's occupancy (at most this
// many entries); a row segment whose list would be longer than that, or than a
// quarter of the segment, takes the passes over the cache.
constexpr int kRowListMax = 3072;

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

// Adds each lane's bin (lanes with `in` set) to a shared-memory histogram.  A
// warp with no lane in skips (most warps, in the passes that filter on a
// prefix); a warp whose lanes all hold the same bin makes one atomic (ties,
// constant rows); otherwise every lane adds its own.
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool in, int lane) {
  const uint32_t inmask = __ballot_sync(0xffffffffu, in);
  if (inmask == 0) return;
  const int leader = __ffs(inmask) - 1;
  const uint32_t b0 = __shfl_sync(0xffffffffu, bin, leader);
  const uint32_t same = __ballot_sync(0xffffffffu, in && bin == b0);
  if (same == inmask) {
    if (lane == leader) atomicAdd(&hist[b0], static_cast<uint32_t>(__popc(inmask)));
  } else if (in) {
    atomicAdd(&hist[bin], 1u);
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
      hist_add(hist, (k[u] >> shift) & mask, in, lane);
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

// Ordered compaction of a cached row segment: the positions of its keys whose
// top 11 bits are >= b1, in index order, into `list`; returns their number.
// One block scan per 2048 keys.
__device__ int compact_at_or_above(const uint32_t* cache, int m, uint32_t b1, int32_t* list, uint32_t* scratch) {
  int out_base = 0;
  for (int base = 0; base < m; base += kStep) {
    const int i = base + threadIdx.x * kPer;
    const uint4 v = *reinterpret_cast<const uint4*>(cache + i);   // the cache is whole steps long
    const uint32_t kk[kPer] = {v.x, v.y, v.z, v.w};
    uint32_t cnt = 0;
    bool f[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      f[u] = (i + u) < m && (kk[u] >> 21) >= b1;
      cnt += f[u] ? 1u : 0u;
    }
    uint32_t total;
    const uint32_t incl = block_scan(cnt, scratch, &total);
    int pos = out_base + static_cast<int>(incl - cnt);
#pragma unroll
    for (int u = 0; u < kPer; ++u)
      if (f[u]) list[pos++] = i + u;
    out_base += static_cast<int>(total);
  }
  return out_base;
}

// hist_pass over the listed keys of a cached row.
__device__ void hist_listed(const uint32_t* cache, const int32_t* list, int m, uint32_t* hist, int shift, int bits,
                            int fshift, uint32_t prefix) {
  const int lane = threadIdx.x & 31;
  const uint32_t mask = (1u << bits) - 1u;
  for (int base = 0; base < m; base += kThreads) {
    const int i = base + threadIdx.x;
    const uint32_t key = i < m ? cache[list[i]] : 0u;
    hist_add(hist, (key >> shift) & mask, i < m && (key >> fshift) == prefix, lane);
  }
}

// Counts of listed keys above / equal to tau.
__device__ void count_listed(const uint32_t* cache, const int32_t* list, int m, uint32_t tau, uint32_t& cgt,
                             uint32_t& ceq) {
  cgt = 0;
  ceq = 0;
  for (int i = threadIdx.x; i < m; i += kThreads) {
    const uint32_t key = cache[list[i]];
    cgt += key > tau ? 1u : 0u;
    ceq += key == tau ? 1u : 0u;
  }
}

// Output pass over the listed keys (index order, four per thread per step):
// every key above tau and the first `need` keys equal to it, at slots after
// gt_base / eq_base earlier ones; `lo` is the global index of the cached
// segment's first key.
__device__ void output_listed(const uint32_t* cache, const int32_t* list, int m, uint32_t tau, uint32_t need, int k,
                              int lo, uint32_t gt_base, uint32_t eq_base, int32_t* out, uint32_t* scratch) {
  for (int base = 0; base < m; base += kStep) {
    const int i = base + threadIdx.x * kPer;
    int pos[kPer];
    uint32_t kk[kPer];
    bool valid[kPer];
    uint32_t cgt = 0, ceq = 0;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      valid[u] = i + u < m;
      pos[u] = valid[u] ? list[i + u] : 0;
      kk[u] = valid[u] ? cache[pos[u]] : 0u;
      cgt += (valid[u] && kk[u] > tau) ? 1u : 0u;
      ceq += (valid[u] && kk[u] == tau) ? 1u : 0u;
    }
    const uint32_t packed = cgt | (ceq << 16);
    uint32_t total;
    const uint32_t excl = block_scan(packed, scratch, &total) - packed;
    uint32_t gt_before = gt_base + (excl & 0xffffu);
    uint32_t eq_before = eq_base + (excl >> 16);
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      if (!valid[u]) continue;
      if (kk[u] > tau) {
        const uint32_t slot = gt_before + min(eq_before, need);
        if (slot < static_cast<uint32_t>(k)) out[slot] = lo + pos[u];
        ++gt_before;
      } else if (kk[u] == tau) {
        const uint32_t slot = gt_before + eq_before;
        if (eq_before < need && slot < static_cast<uint32_t>(k)) out[slot] = lo + pos[u];
        ++eq_before;
      }
    }
    gt_base += total & 0xffffu;
    eq_base += total >> 16;
  }
}

// A list pays when it holds at most a quarter of the segment's keys.
__device__ __forceinline__ bool use_list(uint32_t at_or_above, int list_cap, int m) {
  return at_or_above <= static_cast<uint32_t>(list_cap) && 4u * at_or_above <= static_cast<uint32_t>(m);
}

// Exact top-k of row c (n > k) by three histogram passes (11, 11, 10 key bits)
// and one output pass over the row: from the shared-memory cache when c.cache
// is set (the first pass fills it), from L2 otherwise.  An uncached row whose
// first histogram the indexer already emitted (hist_in) skips the first pass.
__device__ void select_streaming(const Ctx& c, int k, int32_t* out, uint32_t* hist, uint32_t* scratch,
                                 uint32_t* sel, const uint32_t* hist_in, int32_t* list, int list_cap) {
  const bool cached = c.cache != nullptr;
  const int n = c.n;
  // pass 1: bits 31..21
  if (hist_in && !cached) {
    for (int b = threadIdx.x; b < 2048; b += kThreads) hist[b] = __ldg(hist_in + b);
    __syncthreads();
  } else {
    for (int b = threadIdx.x; b < 2048; b += kThreads) hist[b] = 0;
    __syncthreads();
    hist_pass(c, false, cached, hist, 21, 11, 32, 0);
    __syncthreads();
  }
  find_bin(hist, 2048, static_cast<uint32_t>(k), scratch, &sel[0], &sel[1]);
  const uint32_t b1 = sel[0], r1 = sel[1];
  // keys at or above bin b1: the k - r1 above it and the bin's own
  const uint32_t at_or_above = static_cast<uint32_t>(k) - r1 + hist[b1];
  __syncthreads();

  if (cached && list && use_list(at_or_above, list_cap, n)) {
    // the remaining passes and the output over the listed keys only
    const int m = compact_at_or_above(c.cache, n, b1, list, scratch);
    for (int b = threadIdx.x; b < 2048; b += kThreads) hist[b] = 0;
    __syncthreads();
    hist_listed(c.cache, list, m, hist, 10, 11, 21, b1);
    __syncthreads();
    find_bin(hist, 2048, r1, scratch, &sel[0], &sel[1]);
    const uint32_t pre2 = (b1 << 11) | sel[0], r2 = sel[1];
    __syncthreads();
    for (int b = threadIdx.x; b < 1024; b += kThreads) hist[b] = 0;
    __syncthreads();
    hist_listed(c.cache, list, m, hist, 0, 10, 10, pre2);
    __syncthreads();
    find_bin(hist, 1024, r2, scratch, &sel[0], &sel[1]);
    const uint32_t tau = (pre2 << 10) | sel[0], need = sel[1];
    __syncthreads();
    output_listed(c.cache, list, m, tau, need, k, 0, 0u, 0u, out, scratch);
    return;
  }

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

__global__ void __launch_bounds__(kThreads) topk_kernel(TopkParams p, int cache_elems, int list_cap) {
  extern __shared__ __align__(16) uint32_t tk_smem[];
  uint32_t* hist = tk_smem;                 // 2048
  uint32_t* scratch = hist + 2048;          // 32
  uint32_t* sel = scratch + 32;             // [0] bin, [1] remaining
  uint32_t* cache = sel + 32;               // cache_elems (16-byte aligned: offset 2112 words)
  int32_t* list = list_cap > 0 ? reinterpret_cast<int32_t*>(cache + cache_elems) : nullptr;   // list_cap
  const int t = blockIdx.x;
  int32_t* out = p.idx + static_cast<int64_t>(t) * p.k;
  const int n = row_length(p, t, out);
  if (n <= 0) return;
  const Ctx c{p.scores + static_cast<int64_t>(t) * p.ld, n <= cache_elems ? cache : nullptr, n};
  select_streaming(c, p.k, out, hist, scratch, sel, p.hist ? p.hist + static_cast<int64_t>(t) * 2048 : nullptr,
                   list, list_cap);
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
    const uint32_t key = keys[i < m ? i : 0];
    const bool in = i < m && (key >> fshift) == prefix;
    hist_add(hist, (key >> shift) & mask, in, lane);
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
    select_streaming(c, k, out, hist, scratch, sel, nullptr, nullptr, 0);
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

// ---------------------------------------------------------------- few long rows: a cluster per row
// When the rows are few (decode), one CTA per row leaves most SMs idle.  Here a
// cluster of C CTAs (2, 4 or 8) shares a row: CTA r caches the keys of segment r
// (consecutive indices) in its shared memory.  Each radix pass (11, 11 and 10
// key bits) histograms the CTA's segment locally, then adds the non-zero bins
// into every CTA's copy of the cluster histogram (remote reductions through
// distributed shared memory, which need no round trip); after one cluster
// barrier every CTA finds the same threshold bin in its own copy.  The output
// pass writes each CTA's selected keys at the offset given by the selections of
// the segments before it, so the result is in index order with ties going to
// the lower index, as in the single-CTA kernels.  The row is read from memory
// once; five cluster barriers in all.
__device__ __forceinline__ uint32_t cl_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cl_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cl_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t cl_map(const void* p, uint32_t cta) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(cta));
  return r;
}
__device__ __forceinline__ void red_add_cluster(uint32_t addr, uint32_t v) {
  asm volatile("red.relaxed.cluster.shared::cluster.add.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void st_cluster(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

struct ClusterShared {
  uint32_t local[2048];          // this CTA's histogram of the current pass
  uint32_t global[2][2048];      // the cluster's histogram (passes alternate buffers)
  uint32_t scratch[32];
  uint32_t sel[2];
  uint32_t cnt_gt[8], cnt_eq[8]; // per-CTA counts of keys above / equal to the threshold
};

// Adds this CTA's histogram (nbins bins) into every CTA's `global` buffer.
__device__ __forceinline__ void cl_push(const ClusterShared& S, uint32_t* dst, int nbins, uint32_t C) {
  for (int b = threadIdx.x; b < nbins; b += kThreads) {
    const uint32_t v = S.local[b];
    if (v == 0) continue;
    for (uint32_t c = 0; c < C; ++c) red_add_cluster(cl_map(dst + b, c), v);
  }
}

__global__ void __launch_bounds__(kThreads) topk_cluster_kernel(TopkParams p, int seg_cap, int list_cap) {
  extern __shared__ __align__(16) uint32_t tk_smem[];
  ClusterShared& S = *reinterpret_cast<ClusterShared*>(tk_smem);
  uint32_t* cache = tk_smem + (sizeof(ClusterShared) + 15) / 16 * 4;   // seg_cap keys
  int32_t* list = reinterpret_cast<int32_t*>(cache + seg_cap);          // list_cap positions
  const uint32_t C = cl_size(), r = cl_rank();
  const int t = blockIdx.x / static_cast<int>(C);
  const int k = p.k;
  const int lane = threadIdx.x & 31;
  int32_t* out = p.idx + static_cast<int64_t>(t) * k;
  // row length (identical in every CTA of the cluster, so all take the same branches)
  int n = -1;
  {
    const int seq = p.q_seq[t];
    if (seq >= 0 && seq < p.num_seqs) {
      const int len = p.kv_len[seq];
      const int pos = p.q_pos[t];
      if (len >= 0 && len <= p.max_kv_len && pos >= 0 && pos < len) n = pos + 1;
    }
  }
  if (n < 0 || n <= k) {                                   // every CTA writes its share of the row
    if (n < 0 && r == 0 && threadIdx.x == 0) set_status(p.status, DSA_DEV_BAD_QUERY);
    for (int j = static_cast<int>(r) * kThreads + threadIdx.x; j < k; j += static_cast<int>(C) * kThreads)
      out[j] = (j < n) ? j : -1;
    return;
  }
  const int seg = ((n + static_cast<int>(C) - 1) / static_cast<int>(C) + kPer - 1) / kPer * kPer;
  if (seg > seg_cap) {                                     // cannot happen with the host's sizing
    if (r == 0 && threadIdx.x == 0) set_status(p.status, DSA_DEV_INTERNAL);
    for (int j = static_cast<int>(r) * kThreads + threadIdx.x; j < k; j += static_cast<int>(C) * kThreads) out[j] = -1;
    return;
  }
  const int lo = min(n, static_cast<int>(r) * seg);
  const int m = min(n, lo + seg) - lo;                     // keys of this CTA's segment
  const float* row = p.scores + static_cast<int64_t>(t) * p.ld + lo;

  for (int b = threadIdx.x; b < 2048; b += kThreads) {
    S.local[b] = 0;
    S.global[0][b] = 0;
    S.global[1][b] = 0;
  }
  __syncthreads();
  cl_sync();                                               // every copy is cleared before any reduction

  // pass 1: cache the segment's keys and histogram bits 31..21 (unless the
  // indexer emitted the row's histogram); four 16-byte loads per thread in flight
  const bool have_hist = p.hist != nullptr;               // uniform over the grid
  constexpr int kUnroll = 4;
  for (int base = 0; base < m; base += kStep * kUnroll) {
    uint32_t kk[kUnroll][kPer];
#pragma unroll
    for (int w = 0; w < kUnroll; ++w) {
      const int i = base + w * kStep + threadIdx.x * kPer;
      if (i + kPer <= m) {
        const float4 f = __ldg(reinterpret_cast<const float4*>(row + i));   // lo and ld are multiples of 4
        kk[w][0] = order_key(f.x); kk[w][1] = order_key(f.y); kk[w][2] = order_key(f.z); kk[w][3] = order_key(f.w);
      } else {
#pragma unroll
        for (int u = 0; u < kPer; ++u) kk[w][u] = (i + u) < m ? order_key(__ldg(row + i + u)) : 0u;
      }
    }
#pragma unroll
    for (int w = 0; w < kUnroll; ++w) {
      const int i = base + w * kStep + threadIdx.x * kPer;
      if (i < m) *reinterpret_cast<uint4*>(cache + i) = make_uint4(kk[w][0], kk[w][1], kk[w][2], kk[w][3]);
      if (!have_hist) {
#pragma unroll
        for (int u = 0; u < kPer; ++u) hist_add(S.local, kk[w][u] >> 21, (i + u) < m, lane);
      }
    }
  }
  __syncthreads();
  if (have_hist) {
    // every CTA of the cluster reads the same row histogram: no reduction needed
    const uint32_t* hg = p.hist + static_cast<int64_t>(t) * 2048;
    for (int b = threadIdx.x; b < 2048; b += kThreads) S.global[0][b] = __ldg(hg + b);
    __syncthreads();
  } else {
    cl_push(S, S.global[0], 2048, C);
    cl_sync();                                             // the cluster's histogram is complete everywhere
  }
  find_bin(S.global[0], 2048, static_cast<uint32_t>(k), S.scratch, &S.sel[0], &S.sel[1]);
  const uint32_t b1 = S.sel[0], r1 = S.sel[1];
  __syncthreads();

  // This segment's keys at or above bin b1 (from its own pass-1 histogram): when
  // they fit the list, the later passes and the output run over their positions
  // only.  Each CTA decides for itself; the cluster steps below are the same.
  bool listed = false;
  if (!have_hist && list_cap > 0) {                        // uniform over the grid
    uint32_t mine = 0;
    for (int b = threadIdx.x; b < 2048; b += kThreads) mine += b >= static_cast<int>(b1) ? S.local[b] : 0u;
    uint32_t at_or_above;
    block_scan(mine, S.scratch, &at_or_above);
    listed = use_list(at_or_above, list_cap, m);
  }
  const int ml = listed ? compact_at_or_above(cache, m, b1, list, S.scratch) : 0;

  // pass 2: bits 20..10 of the keys with the pass-1 prefix (global[1] was cleared at the start)
  for (int b = threadIdx.x; b < 2048; b += kThreads) {
    S.local[b] = 0;
    S.global[0][b] = 0;                                    // read above; peers write it again only after the next barrier
  }
  __syncthreads();
  const Ctx cc{nullptr, cache, m};
  if (listed) hist_listed(cache, list, ml, S.local, 10, 11, 21, b1);
  else hist_pass(cc, true, false, S.local, 10, 11, 21, b1);
  __syncthreads();
  cl_push(S, S.global[1], 2048, C);
  cl_sync();
  find_bin(S.global[1], 2048, r1, S.scratch, &S.sel[0], &S.sel[1]);
  const uint32_t b2 = S.sel[0], r2 = S.sel[1];
  __syncthreads();

  // pass 3: bits 9..0
  const uint32_t pre2 = (b1 << 11) | b2;
  for (int b = threadIdx.x; b < 2048; b += kThreads) S.local[b] = 0;
  __syncthreads();
  if (listed) hist_listed(cache, list, ml, S.local, 0, 10, 10, pre2);
  else hist_pass(cc, true, false, S.local, 0, 10, 10, pre2);
  __syncthreads();
  cl_push(S, S.global[0], 1024, C);
  cl_sync();
  find_bin(S.global[0], 1024, r2, S.scratch, &S.sel[0], &S.sel[1]);
  const uint32_t tau = (pre2 << 10) | S.sel[0];            // the k-th largest key
  const uint32_t need = S.sel[1];                          // its copies to take, lowest indices first
  __syncthreads();

  // counts above / equal to tau of every segment -> offsets of this segment's output
  {
    uint32_t cgt = 0, ceq = 0;
    if (listed) {
      count_listed(cache, list, ml, tau, cgt, ceq);
    } else {
      for (int i = threadIdx.x; i < m; i += kThreads) {
        const uint32_t key = cache[i];
        cgt += key > tau ? 1u : 0u;
        ceq += key == tau ? 1u : 0u;
      }
    }
    uint32_t tgt, teq;
    block_scan(cgt, S.scratch, &tgt);
    block_scan(ceq, S.scratch, &teq);
    if (threadIdx.x < static_cast<int>(C)) {
      st_cluster(cl_map(&S.cnt_gt[r], threadIdx.x), tgt);
      st_cluster(cl_map(&S.cnt_eq[r], threadIdx.x), teq);
    }
  }
  cl_sync();                                               // last access to another CTA's memory
  uint32_t gt_base = 0, eq_base = 0;
  for (uint32_t c = 0; c < r; ++c) { gt_base += S.cnt_gt[c]; eq_base += S.cnt_eq[c]; }
  if (listed) {
    output_listed(cache, list, ml, tau, need, k, lo, gt_base, eq_base, out, S.scratch);
    return;
  }

  // output pass over the cached segment, index order (global index = lo + i)
  for (int base = 0; base < m; base += kStep) {
    const int i = base + threadIdx.x * kPer;
    uint32_t kk[kPer];
    bool valid[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      valid[u] = i + u < m;
      kk[u] = valid[u] ? cache[i + u] : 0u;
    }
    uint32_t cgt = 0, ceq = 0;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      cgt += (valid[u] && kk[u] > tau) ? 1u : 0u;
      ceq += (valid[u] && kk[u] == tau) ? 1u : 0u;
    }
    const uint32_t packed = cgt | (ceq << 16);
    uint32_t total;
    const uint32_t incl = block_scan(packed, S.scratch, &total);
    const uint32_t excl = incl - packed;
    uint32_t gt_before = gt_base + (excl & 0xffffu);
    uint32_t eq_before = eq_base + (excl >> 16);
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      if (!valid[u]) continue;
      if (kk[u] > tau) {
        const uint32_t slot = gt_before + min(eq_before, need);
        if (slot < static_cast<uint32_t>(k)) out[slot] = lo + i + u;
        ++gt_before;
      } else if (kk[u] == tau) {
        const uint32_t slot = gt_before + eq_before;
        if (eq_before < need && slot < static_cast<uint32_t>(k)) out[slot] = lo + i + u;
        ++eq_before;
      }
    }
    gt_base += total & 0xffffu;
    eq_base += total >> 16;
  }
}

}  // namespace

// Which kernel launch_topk picks for these rows: 2..8 = a cluster of that many
// CTAs per row, 1 = the two-read long-row kernel, 0 = the streaming kernel with
// rows cached in shared memory, -1 = the streaming kernel reading rows from L2.
int topk_plan(int max_kv_len, int T, int sms) {
  if (max_kv_len >= kClusterMinLen) {
    auto seg_of = [&](int c) { return (((max_kv_len + c - 1) / c + kStep - 1) / kStep) * kStep; };
    int c_fit = 1;
    while (c_fit <= 8 && seg_of(c_fit) > kClusterSegMax) c_fit <<= 1;
    int c_par = 8;
    while (c_par > 1 && T * c_par > 2 * sms) c_par >>= 1;
    const int C = c_fit > c_par ? c_fit : c_par;
    if (C >= 2 && C <= 8) return C;
  }
  const int cache_elems = ((max_kv_len + kStep - 1) / kStep) * kStep;
  if (cache_elems > kCacheMax && T <= 2 * sms) return 1;
  return cache_elems > kCacheMax ? -1 : 0;
}

bool topk_uses_hist(int max_kv_len, int T, int sms) {
  const int plan = topk_plan(max_kv_len, T, sms);
  return plan >= 2 || plan == -1;
}

// A list is allocated only for rows of at least 5k keys (it must stay within a
// quarter of them) and, in a cluster, only when it can hold a segment's share of
// about 1.5k keys.
// Entries of a row list that fit in the shared memory a CTA of `base` bytes
// leaves over at its occupancy without one (at most four 512-thread CTAs per
// SM); 0 when fewer than 512 fit.
int list_cap_for(size_t base, int dev) {
  int per_sm = 0, reserved = 0, per_block = 0;
  if (cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&per_block, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return 0;
  const size_t slot = base + static_cast<size_t>(reserved);
  size_t ctas = static_cast<size_t>(per_sm) / slot;
  if (ctas == 0) return 0;
  if (ctas > 4) ctas = 4;
  size_t room = static_cast<size_t>(per_sm) / ctas - slot;
  if (base + room > static_cast<size_t>(per_block)) room = base < static_cast<size_t>(per_block) ? per_block - base : 0;
  size_t cap = room / sizeof(int32_t) / 4 * 4;
  if (cap > static_cast<size_t>(kRowListMax)) cap = kRowListMax;
  return cap >= 512 ? static_cast<int>(cap) : 0;
}

cudaError_t launch_topk(const TopkParams& p, int T, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  int cache_elems = ((p.max_kv_len + kStep - 1) / kStep) * kStep;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess)
    sms = 148;
  // A cluster of C CTAs per row (C in 2, 4, 8), each caching one segment, when
  // the rows are too long for one CTA's cache (C = the fewest CTAs whose
  // segments fit) or too few to fill the SMs (C = the most CTAs that keep the
  // grid within two per SM).
  if (p.max_kv_len >= kClusterMinLen) {
    // segment cache, rounded up to whole block steps: the passes over it read in steps of kStep keys
    auto seg_of = [&](int c) { return (((p.max_kv_len + c - 1) / c + kStep - 1) / kStep) * kStep; };
    int c_fit = 1;
    while (c_fit <= 8 && seg_of(c_fit) > kClusterSegMax) c_fit <<= 1;
    int c_par = 8;
    while (c_par > 1 && T * c_par > 2 * sms) c_par >>= 1;
    const int C = c_fit > c_par ? c_fit : c_par;
    if (C >= 2 && C <= 8) {
      const int seg_cap = seg_of(C);
      const size_t base = (sizeof(ClusterShared) + 15) / 16 * 16 + static_cast<size_t>(seg_cap) * sizeof(uint32_t);
      // a segment's list holds about (k + one bin) / C keys
      int list_cap = p.max_kv_len >= 5 * p.k ? list_cap_for(base, dev) : 0;
      if (list_cap < (3 * p.k / 2 + C - 1) / C) list_cap = 0;
      const size_t smem = base + static_cast<size_t>(list_cap) * sizeof(int32_t);
      cudaError_t e = cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
      if (e != cudaSuccess) return e;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(static_cast<unsigned>(T * C));
      cfg.blockDim = dim3(kThreads);
      cfg.dynamicSmemBytes = smem;
      cfg.stream = stream;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = static_cast<unsigned>(C);
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      e = cudaLaunchKernelEx(&cfg, topk_cluster_kernel, p, seg_cap, list_cap);
      if (e == cudaSuccess) count_launches(1);
      return e;
    }
  }
  // Rows longer than eight segments.  With few rows (at most two per SM) each CTA
  // has an SM to itself and reading the row twice instead of four times wins;
  // with many rows the streaming kernel, four CTAs per SM, keeps more loads in
  // flight.
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
  const size_t base = (2048 + 64) * sizeof(uint32_t) + static_cast<size_t>(cache_elems) * sizeof(uint32_t);
  const int list_cap = cache_elems > 0 && p.max_kv_len >= 5 * p.k ? list_cap_for(base, dev) : 0;
  const size_t smem = base + static_cast<size_t>(list_cap) * sizeof(int32_t);
  cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  topk_kernel<<<T, kThreads, smem, stream>>>(p, cache_elems, list_cap);
  e = cudaGetLastError();
  if (e == cudaSuccess) count_launches(1);
  return e;
}

}  // namespace dsa
