// Sparse MLA in MQA form on sm_100a.
//
// Page "一文讀懂DeepSeek-V3.2核心技術DSA", "DSA 的四步工作流程" step 4: attention
// over only the selected tokens; page "DeepSeek-V3.2加速技术详解" 3.1 (MQA form of
// MLA: every head attends to the shared latent row, the value is the latent,
// restored afterwards) and 3.2 (unselected tokens are dropped); page "DeepSeek
// 稀疏注意力路线", "工程要点" (the top-k index list makes the KV gather irregular).
//
// Per query token the state is large: Q is 128 heads x 576 (144 KB bf16) and
// the output accumulator 128 x 512 fp32 (256 KB, all of one SM's TMEM).  So a
// token is handled by a CTA pair (a 2-CTA cluster) using the pair form of the
// tensor-core MMA (cta_group::2, M = 128 = 64 heads per CTA), over blocks of
// 256 selected rows, 128 gathered by each CTA:
//   S  = Q K^T : A = the CTA's 64 heads of Q (72 KB, resident), B = the block's
//                256 rows (K-major), N = 256; per CTA: 64 heads x 256 rows fp32
//                in TMEM (128 columns).
//   O += P V   : A = P (64 heads x 256 rows, bf16, K-major, written by the
//                softmax warps), B = V rows of the block, each CTA holding 128
//                of every 256 value dims (MN-major), N = 256; per CTA: 64 heads
//                x 512 dims fp32 (256 TMEM columns).
// A pair MMA with N = 128 takes about as long as one with N = 256 (measured
// 35.5 vs 36.7 ns), so the block is 256 rows wide: every S and PV instruction
// moves 64 x 256 per SM, and a block needs 68 of them.  S is double buffered in
// TMEM, so the tensor core computes S of block j+1 while the softmax warps turn
// S of block j into P.  The softmax keeps a reference maximum per head and
// rescales O (in TMEM) only when a block's maximum exceeds it by more than 2^8,
// so P stays <= 256 and most blocks skip the rescale.
//
// Persistent pairs: a pair walks the items (query, split) cid, cid + pairs, ...;
// the rings and the per-block barriers count across items, so the next query's
// index scan, gathers, Q load and first S MMAs overlap the current query's last
// softmax, PV and output.
//
// Rows are gathered from L2 by index with 16-byte cp.async (8 lanes per 128-byte
// row segment: coalesced) into 128-byte-swizzled tiles.  Two streaming rings
// decouple the gathers from the MMAs: the S ring holds 64-dim chunks of the
// CTA's 128 rows (16 KB slots, refilled as soon as the S MMAs read them) and
// the V ring holds 32-row slices of the block with the CTA's value dims (16 KB
// slots, refilled as soon as the PV MMAs read them).  Each CTA thus reads the
// value dims it multiplies straight from L2; no V data crosses the pair.  The
// gathers' shared-memory writes and the MMAs' operand reads share the SM's
// shared-memory bandwidth (measured: gathers alone 73 B/clk, with back-to-back
// MMAs 41 B/clk while the MMAs slow from 128 to 160 clk each).
//
// Warps: 0-3 softmax / output (TMEM lane quadrants 0-3), 4-11 index scans and
// gathers of the S ring, 12-19 gathers of the V ring, 20 TMEM owner, Q loads
// (both CTAs) and (in the even CTA) issuer of the S MMAs, 21 S relay, 22 V
// relay, 23 (even CTA) issuer of the PV MMAs.  Sixteen gather warps: one SM's
// 16-byte cp.async gathers from L2 scale with the number of warps issuing them
// (about 27 B/clk with eight, 42 with sixteen).  Signals from the odd CTA to
// the even CTA's barriers are asynchronous 4-byte stores counted as transaction
// bytes (a thread-level remote mbarrier arrive stalls its thread for a round
// trip).  Gather threads never wait for their own copies: each arrives on a
// local stage barrier through cp.async.mbarrier.arrive (hardware-tracked
// completion), and a relay lane that has no copies in flight forwards the
// completed stage to the even CTA's barrier, which the MMA issuer waits on.
#include <cuda_bf16.h>

#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {

namespace {

constexpr int kMlaThreads = 768;
constexpr int kSWarps = 8;            // S-ring gather warps: 16 rows of every chunk each
constexpr int kVWarps = 8;            // V-ring gather warps: 4 rows of every slice each
constexpr int kRoleWarp = 4 + kSWarps + kVWarps;   // first of the four single-lane role warps
// Registers: launched at 80 per thread (768 x 80 = 61,440); the softmax
// warpgroup takes 160, every other warpgroup gives back down to 64
// (128 x 160 + 640 x 64 = 61,440).
// Readers of a plan slot that release it (plan_free), one arrival each: the 4
// softmax warps, the 16 gather warps and three single-lane roles (plus the PV
// issuer in the even CTA).
constexpr uint32_t kPlanReaders = 4 + kSWarps + kVWarps + 3;
constexpr uint32_t kLaunchRegs = 80;
constexpr uint32_t kRegsSoftmax = 160;
constexpr uint32_t kRegsOther = 64;
static_assert(128 * kRegsSoftmax + (kMlaThreads - 128) * kRegsOther == kMlaThreads * kLaunchRegs,
              "the register split must add up to the launch allocation");
constexpr int kBlk = 256;             // selected rows per block (pair)
constexpr int kRows = 128;            // rows per CTA per block (S operand)
constexpr int kHeads = 64;            // heads per CTA
constexpr int kDChunks = DSA_D_QK / 64;   // 9 chunks of 64 dims
constexpr int kSStages = 3;           // S ring: 16 KB slots (128 rows x 64 dims)
constexpr int kVRows = 32;            // rows per V slice
constexpr int kVSlices = kBlk / kVRows;   // 8 slices per block
constexpr int kVStages = 4;           // V ring: 16 KB slots (32 rows x 256 value dims)
constexpr float kRescaleThreshold = 8.0f;   // log2 units
constexpr uint32_t kSCol = 0;         // TMEM columns [0,256): two S buffers of 128
constexpr uint32_t kOCol = 256;       // TMEM columns [256,512): O (2 x 128)

struct MlaSmem {
  uint8_t q[kDChunks][kHeads * 128];         // 72 KB  Q of this CTA's heads (K-major SW128)
  uint8_t s_ring[kSStages][kRows * 128];     // 48 KB  S operand chunks: 128 rows x 64 dims
  uint8_t v_ring[kVStages][4][kVRows * 128]; // 64 KB  V slices: 4 dim groups x 32 rows (MN-major SW128)
  uint8_t p[kBlk / 64][kHeads * 128];        // 32 KB  P: 64 heads x 256 rows (four K chunks of 64 rows)
  float xmax[2][128];
  float lsum[128];
  uint32_t valid[2][2048 / 32];              // per plan slot: bit e = entry e of the index row is usable
  int last_used[2][kSWarps];                 // per plan slot and scanning warp: last usable entry, -1 if none
  uint64_t q_full, q_ready, q_empty;
  uint64_t s_full[kSStages], s_empty[kSStages], s_loaded[kSStages];
  uint64_t v_full[kVStages], v_empty[kVStages], v_loaded[kVStages];
  uint64_t s_ready[2], s_free[2];
  uint64_t p_full[2], p_empty[2];            // per half of P: rows 0..127 (chunks 0-1), 128..255 (chunks 2-3)
  uint64_t mx_bar[2], l_bar;
  uint64_t o_done[2];                         // O lanes of warp 2+i rescaled (local, for warp i)
  uint64_t o_full;                            // the last PV MMAs of a query completed (both CTAs)
  uint64_t o_free;                            // (even CTA) both CTAs' epilogues have read O out
  uint64_t plan_ready[2], plan_free[2];       // per plan slot: written by the scanners / released by its readers
  uint64_t done;
  // mailboxes of the peer CTA's asynchronous signals (contents unused)
  uint32_t mbox_q, mbox_s[kSStages], mbox_v[kVStages], mbox_sfree[2][4], mbox_pfull[2][2], mbox_ofree[4];
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// No memory clobber: the copies are ordered against their consumers by mbarriers,
// and leaving the compiler free to schedule address arithmetic keeps the gather
// warps issuing back to back.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// Arrive on `bar` once every cp.async issued so far by this thread has completed.
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Cross-CTA signalling convention for barriers of the even CTA that wait on both
// CTAs: the even CTA arrives locally (one arrival carrying expect_tx for the odd
// CTA's bytes), the odd CTA sends 4-byte asynchronous stores (st_async_signal).
__device__ __forceinline__ void pair_signal(uint32_t rank, uint64_t* bar, uint32_t* mbox, bool carries_tx,
                                            uint32_t tx_bytes) {
  if (rank == 0) {
    if (carries_tx) mbar_arrive_expect_tx(bar, tx_bytes);
    else mbar_arrive(bar);
  } else {
    st_async_signal(mbox, bar, 0, 1u);
  }
}

// Lane-0 waits, the warp follows (warp-uniform result).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint32_t* status, volatile int* ab,
                                          bool cluster_scope) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0)
    ok = (cluster_scope ? mbar_wait_cluster(bar, parity, status, ab) : mbar_wait(bar, parity, status, ab)) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// Order in which the chunks of a block are gathered, forwarded and multiplied:
// the RoPE chunk (dims 512..575) first, then the value chunks 0..7.
__device__ __forceinline__ int chunk_at(int i) { return i == 0 ? kDChunks - 1 : i - 1; }

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kMlaThreads, 1)
sparse_mla_kernel(const __grid_constant__ CUtensorMap tm_q, MlaParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  MlaSmem& S = *reinterpret_cast<MlaSmem*>(smem_raw);   // 1024-aligned: checked below
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  // Persistent pairs: pair `cid` takes the items (query, split) cid, cid + ncl, ...
  // Every role walks the same item sequence; the rings and the per-block
  // barriers keep counting across items, so the gathers and S MMAs of the next
  // query overlap the softmax, PV and output of the current one.
  const int cid = blockIdx.x >> 1;
  const int ncl = static_cast<int>(gridDim.x >> 1);
  const int n_items = p.T * p.splits;
  volatile int* ab = &S.abort_flag;
  const int H = p.H;
  const int head0 = static_cast<int>(rank) * kHeads;       // first head of this CTA

  struct Item {
    int t, split, seq, len;
    int64_t base;
    bool ok;
    const int32_t* idx_row;
  };
  // per-query facts (identical in both CTAs)
  auto item_of = [&](int it) {
    Item I;
    I.t = it / p.splits;
    I.split = it % p.splits;
    const int seq = p.q_seq[I.t];
    const bool seq_ok = seq >= 0 && seq < p.num_seqs;
    I.seq = seq_ok ? seq : 0;
    I.len = seq_ok ? p.kv_len[seq] : 0;
    I.base = seq_ok && p.page_size == 0 ? p.kv_offset[seq] : 0;
    I.ok = seq_ok && I.len >= 0 &&
           (p.page_size == 0 ? I.base >= 0 && I.base + I.len <= p.kv_rows
                             : I.len <= static_cast<int64_t>(p.pages_per_seq) * p.page_size);
    I.idx_row = p.idx + static_cast<int64_t>(I.t) * p.k;
    return I;
  };
  // cache row of the usable local index v (0 <= v < len), -1 (flagged) when its
  // page points outside the cache
  auto cache_row = [&](const Item& I, int v) -> int64_t {
    if (p.page_size == 0) return I.base + v;
    const int pg = __ldg(p.page_table + static_cast<int64_t>(I.seq) * p.pages_per_seq + v / p.page_size);
    const int64_t r = static_cast<int64_t>(pg) * p.page_size + v % p.page_size;
    if (pg < 0 || r >= p.kv_rows) {
      set_status(p.status, DSA_DEV_BAD_INDEX);
      return -1;
    }
    return r;
  };
  // blocks of 256 entries covering the used part of the index row, split evenly
  auto plan_of = [&](int b, int split, int& blk0, int& nblk) {
    int last = -1;
#pragma unroll
    for (int w = 0; w < kSWarps; ++w) last = max(last, S.last_used[b][w]);
    const int total = (last + kBlk) / kBlk;
    const int per = (total + p.splits - 1) / p.splits;
    blk0 = min(total, split * per);
    nblk = *ab ? 0 : min(total, blk0 + per) - blk0;
  };

  if (threadIdx.x == 0) {
    mbar_init(&S.q_full, 1);
    mbar_init(&S.q_ready, 1);
    mbar_init(&S.q_empty, 1);
    for (int i = 0; i < kSStages; ++i) {
      mbar_init(&S.s_full[i], 1); mbar_init(&S.s_empty[i], 1); mbar_init(&S.s_loaded[i], kSWarps * 32);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&S.v_full[i], 1); mbar_init(&S.v_empty[i], 1); mbar_init(&S.v_loaded[i], kVWarps * 32);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.s_ready[i], 1); mbar_init(&S.s_free[i], 4); mbar_init(&S.mx_bar[i], 4);
      mbar_init(&S.plan_ready[i], kSWarps); mbar_init(&S.plan_free[i], kPlanReaders + (rank == 0 ? 1 : 0));
    }
    for (int h = 0; h < 2; ++h) { mbar_init(&S.p_full[h], 2); mbar_init(&S.p_empty[h], 1); }
    mbar_init(&S.l_bar, 4);
    mbar_init(&S.o_done[0], 1); mbar_init(&S.o_done[1], 1);
    mbar_init(&S.o_full, 1);
    mbar_init(&S.o_free, 4);
    mbar_init(&S.done, 2);                      // one drain commit per MMA issuer
    S.abort_flag = 0;
    if (smem_u32(smem_raw) & 1023u) {           // the swizzled tiles need 1024-byte alignment
      set_status(p.status, DSA_DEV_INTERNAL);
      S.abort_flag = 1;
    }
    fence_mbar_init();
  }
  if (warp == kRoleWarp) tmem_alloc_pair(&S.tmem_base, 512);
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  if (warp < 4) setmaxnreg_inc<kRegsSoftmax>();
  else setmaxnreg_dec<kRegsOther>();

  if (warp < 4) {
    // ================================================================ softmax
    // Thread = TMEM lane: head hl of this CTA, over the 128 rows gathered by
    // CTA `half` (the S tile's columns 128*half .. +127 sit on lanes 64*half ..).
    const int tid = threadIdx.x;
    const int hl = tid & 63;
    const int half = tid >> 6;
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    int gb = 0;                                            // blocks so far, all items
    uint32_t ne = 0;                                       // items with blocks so far
    uint32_t n_rescaled = 0;                               // blocks j > 0 that rescaled O (this warp)
    bool ok = true;
    for (int kk = 0, it = cid; it < n_items && ok; ++kk, it += ncl) {
      const int b = kk & 1;
      if (!warp_wait(&S.plan_ready[b], (kk >> 1) & 1, p.status, ab, false)) break;
      const Item I = item_of(it);
      int blk0, nblk;
      plan_of(b, I.split, blk0, nblk);
      const int h = head0 + hl;
      const bool store = h < H;                            // TMEM loads stay warp-collective
      if (nblk == 0) {
        // no selected row: output zeros, lse = -inf
        if (store) {
          if (p.splits == 1) {
            uint16_t* orow = p.out + (static_cast<int64_t>(I.t) * H + h) * DSA_D_V;
            for (int d = half * 256; d < half * 256 + 256; d += 8)
              *reinterpret_cast<uint4*>(orow + d) = make_uint4(0, 0, 0, 0);
            if (half == 0 && p.lse) p.lse[static_cast<int64_t>(I.t) * H + h] = -INFINITY;
          } else {
            float* orow = p.part_o + ((static_cast<int64_t>(I.t) * p.splits + I.split) * H + h) * DSA_D_V;
            for (int d = half * 256; d < half * 256 + 256; d += 4)
              *reinterpret_cast<float4*>(orow + d) = make_float4(0.f, 0.f, 0.f, 0.f);
            if (half == 0) p.part_lse[(static_cast<int64_t>(I.t) * p.splits + I.split) * H + h] = -INFINITY;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.plan_free[b]);
        continue;
      }
      float m_ref = -INFINITY, l = 0.f;
      for (int j = 0; j < nblk; ++j, ++gb) {
        const int sb = gb & 1;
        const uint32_t sph = (gb >> 1) & 1;
        // validity of this thread's 128 entries (four 32-bit words)
        const int pos0 = (blk0 + j) * kBlk + half * kRows;   // multiple of 128
        auto valid_word = [&](int c) -> uint32_t { return pos0 + 32 * c < 2048 ? S.valid[b][(pos0 >> 5) + c] : 0u; };
        if (!warp_wait(&S.s_ready[sb], sph, p.status, ab, false)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sbase = tmem + lane_addr + kSCol + sb * 128;
        // pass 1: this thread's maximum over its 128 logits (log2 units)
        float mloc = -INFINITY;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t sr[32];
          tmem_ld32(sbase + c * 32, sr);
          const uint32_t vmc = valid_word(c);
          tmem_ld_wait();
#pragma unroll
          for (int u = 0; u < 32; ++u)
            if ((vmc >> u) & 1u) mloc = fmaxf(mloc, __uint_as_float(sr[u]) * p.sm_scale_log2);
        }
        // pair maximum of this head over the whole block
        S.xmax[sb][tid] = mloc;
        __syncwarp();                                      // one arrival per warp (count 4)
        if (lane == 0) mbar_arrive(&S.mx_bar[sb]);
        if (!warp_wait(&S.mx_bar[sb], sph, p.status, ab, false)) { ok = false; break; }
        const float mblk = fmaxf(mloc, S.xmax[sb][tid ^ 64]);
        const bool rescale = mblk > m_ref + kRescaleThreshold;
        const float m_new = rescale ? mblk : m_ref;
        // a head with no usable entry so far has m_new = -inf and every x = -inf:
        // subtract 0 instead, so that each p is 2^-inf = 0 (never -inf - -inf)
        const float msub = m_new == -INFINITY ? 0.f : m_new;
        const float alpha = rescale ? ex2_approx(m_ref - m_new) : 1.f;   // m_ref = -inf -> 0
        // O is rescaled only from the second block of a query on (the first PV
        // of a query overwrites O); warp-uniform, as TMEM ld/st are warp-collective
        const bool rs_wait = j > 0 && __any_sync(0xffffffffu, rescale);
        // pass 2: P = 2^(x - m) in bf16, held in registers (64 packed pairs) so
        // that the S buffer is released before the P buffer is free; the
        // denominator sums the same bf16 values that the PV MMA multiplies V by
        float psum = 0.f;
        uint32_t pk[64];
#pragma unroll
        for (int c = 0; c < 8; ++c) {                         // 16 columns at a time
          uint32_t sr[16];
          tmem_ld16(sbase + c * 16, sr);
          const uint32_t vmc = valid_word(c >> 1) >> ((c & 1) * 16);
          tmem_ld_wait();
#pragma unroll
          for (int u = 0; u < 16; u += 2) {
            const float x0 = ((vmc >> u) & 1u) ? __uint_as_float(sr[u]) * p.sm_scale_log2 : -INFINITY;
            const float x1 = ((vmc >> (u + 1)) & 1u) ? __uint_as_float(sr[u + 1]) * p.sm_scale_log2 : -INFINITY;
            const uint32_t pp = pack_bf16(ex2_approx(x0 - msub), ex2_approx(x1 - msub));
            psum += __uint_as_float(pp << 16) + __uint_as_float(pp & 0xffff0000u);
            pk[c * 8 + (u >> 1)] = pp;
          }
        }
        l = l * alpha + psum;
        m_ref = m_new;
        // S buffer sb has been read: the S MMAs of block gb+2 may overwrite it
        tc_fence_before();
        __syncwarp();
        if (lane == 0) pair_signal(rank, &S.s_free[sb], &S.mbox_sfree[sb][warp], warp == 0, 16);
        // This thread's half of P (rows 128*half ..) is free once the PV MMAs of
        // the previous block on it completed: the PV consumes rows 0..127 first,
        // so half 0 stores while the PV still multiplies the other half.  O may
        // be rescaled only once the whole previous PV completed.  Warps w and w+2
        // hold the same heads, so they take the same rescale decision; the PV of
        // this block starts on half 0's signal, so warp w then also waits for
        // warp w+2 to have rescaled its O lanes before it signals.
        if (gb > 0) {
          // every block waits for its own half in order (a parity wait must not
          // skip a phase); a rescale also needs the whole previous PV
          if (!warp_wait(&S.p_empty[half], (gb - 1) & 1, p.status, ab, false) ||
              (rs_wait && half == 0 && !warp_wait(&S.p_empty[1], (gb - 1) & 1, p.status, ab, false))) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (rs_wait) {
#pragma unroll 1
            for (int c = 0; c < 16; ++c) {
              uint32_t o[16];
              const uint32_t a = tmem + lane_addr + kOCol + c * 16;
              tmem_ld16(a, o);
              tmem_ld_wait();
#pragma unroll
              for (int u = 0; u < 16; ++u) o[u] = __float_as_uint(__uint_as_float(o[u]) * alpha);
              tmem_st16(a, o);
            }
            tmem_st_wait();
            if (half == 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&S.o_done[warp & 1]);
            }
          }
        }
        // P row hl of K chunks 2*half and 2*half+1 (rows 128*half .. +127 of the
        // block), 128B-swizzled
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint8_t* prow = S.p[half * 2 + (c >> 1)] + hl * 128;
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const int c16 = (c & 1) * 4 + q4;                // 16-byte chunk of the 128-byte row
            *reinterpret_cast<uint4*>(prow + ((c16 ^ (hl & 7)) << 4)) =
                make_uint4(pk[c * 16 + q4 * 4 + 0], pk[c * 16 + q4 * 4 + 1], pk[c * 16 + q4 * 4 + 2],
                           pk[c * 16 + q4 * 4 + 3]);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (half == 0 && rs_wait) {
          if (!warp_wait(&S.o_done[warp & 1], n_rescaled & 1, p.status, ab, false)) { ok = false; break; }
          tc_fence_after();
          tc_fence_before();
        }
        if (rs_wait) ++n_rescaled;
        // per half: warps 2*half, 2*half+1 of both CTAs (the even one's first warp
        // carries the odd CTA's 8 bytes)
        if (lane == 0) pair_signal(rank, &S.p_full[half], &S.mbox_pfull[half][warp & 1], (warp & 1) == 0, 8);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.plan_free[b]);       // this query's validity words are no longer read
      if (!ok) break;
      // ---- epilogue: wait for the last PV, combine the two row halves, write out,
      // then release O to the PV MMAs of the next query
      if (!warp_wait(&S.o_full, ne & 1, p.status, ab, false)) break;
      tc_fence_after();
      S.lsum[tid] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.l_bar);
      if (!warp_wait(&S.l_bar, ne & 1, p.status, ab, false)) break;
      const float lt = l + S.lsum[tid ^ 64];
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      const float lse_v = lt > 0.f ? (m_ref + __log2f(lt)) * 0.69314718055994531f : -INFINITY;
      if (p.splits == 1) {
        uint16_t* orow = p.out + (static_cast<int64_t>(I.t) * H + (store ? h : 0)) * DSA_D_V;
#pragma unroll 1
        for (int c = 0; c < 16; ++c) {
          uint32_t o[16];
          tmem_ld16(tmem + lane_addr + kOCol + c * 16, o);
          tmem_ld_wait();
          const int d0 = (c >> 3) * 256 + half * 128 + (c & 7) * 16;
          uint32_t pkd[8];
#pragma unroll
          for (int u = 0; u < 8; ++u)
            pkd[u] = pack_bf16(__uint_as_float(o[2 * u]) * inv, __uint_as_float(o[2 * u + 1]) * inv);
          if (store) {
            uint4* dst = reinterpret_cast<uint4*>(orow + d0);
            dst[0] = make_uint4(pkd[0], pkd[1], pkd[2], pkd[3]);
            dst[1] = make_uint4(pkd[4], pkd[5], pkd[6], pkd[7]);
          }
        }
        if (store && half == 0 && p.lse) p.lse[static_cast<int64_t>(I.t) * H + h] = lse_v;
      } else {
        float* orow = p.part_o + ((static_cast<int64_t>(I.t) * p.splits + I.split) * H + (store ? h : 0)) * DSA_D_V;
#pragma unroll 1
        for (int c = 0; c < 16; ++c) {
          uint32_t o[16];
          tmem_ld16(tmem + lane_addr + kOCol + c * 16, o);
          tmem_ld_wait();
          const int d0 = (c >> 3) * 256 + half * 128 + (c & 7) * 16;
          if (store) {
            float4* dst = reinterpret_cast<float4*>(orow + d0);
#pragma unroll
            for (int u = 0; u < 4; ++u)
              dst[u] = make_float4(__uint_as_float(o[4 * u]) * inv, __uint_as_float(o[4 * u + 1]) * inv,
                                   __uint_as_float(o[4 * u + 2]) * inv, __uint_as_float(o[4 * u + 3]) * inv);
          }
        }
        if (store && half == 0)
          p.part_lse[(static_cast<int64_t>(I.t) * p.splits + I.split) * H + h] = lse_v;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) pair_signal(rank, &S.o_free, &S.mbox_ofree[warp], warp == 0, 16);
      ++ne;
    }
  } else if (warp < 4 + kSWarps) {
    // ================================================================ S gathers
    // Warps 4-11 first scan the index row of a query (its validity bitmask and
    // last usable entry, into the plan slot of that query), then fill the S
    // ring, chunk by chunk in chunk_at order: warp w loads rows 16w..16w+15 of
    // this CTA's 128 (four 16-byte copies per lane per chunk, 8 lanes per
    // 128-byte row segment) and every lane signals with one hardware-tracked
    // arrive.  A slot is refilled as soon as the S MMAs have read it.  The next
    // query's scan follows the last gathers of the current one.
    const int gw = warp - 4;
    const int c16 = lane & 7;
    const int rsub = lane >> 3;
    auto scan = [&](int kk, int it) -> bool {
      const int b = kk & 1;
      if (kk >= 2 && !warp_wait(&S.plan_free[b], ((kk >> 1) & 1) ^ 1, p.status, ab, false)) return false;
      const Item I = item_of(it);
      if (!I.ok && gw == 0 && lane == 0) set_status(p.status, DSA_DEV_BAD_QUERY);
      int v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = (gw * 8 + u) * 32 + lane;
        v[u] = (I.ok && i < p.k) ? __ldg(I.idx_row + i) : -1;
      }
      int last = -1;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = (gw * 8 + u) * 32 + lane;
        if (v[u] >= I.len) { set_status(p.status, DSA_DEV_BAD_INDEX); v[u] = -1; }
        if (v[u] >= 0) last = i;
        const uint32_t m = __ballot_sync(0xffffffffu, v[u] >= 0);
        if (lane == 0) S.valid[b][gw * 8 + u] = m;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
      if (lane == 0) S.last_used[b][gw] = last;
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.plan_ready[b]);
      return true;
    };
    bool ok = cid < n_items ? scan(0, cid) : true;
    int slot = 0;
    uint32_t sph = 0;
    for (int kk = 0, it = cid; it < n_items && ok; ++kk, it += ncl) {
      const int b = kk & 1;
      if (!warp_wait(&S.plan_ready[b], (kk >> 1) & 1, p.status, ab, false)) break;
      const Item I = item_of(it);
      int blk0, nblk;
      plan_of(b, I.split, blk0, nblk);
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.plan_free[b]);
      // cache rows of this lane's rows (16gw + 4i + rsub) of block bk, -1 if unusable
      auto rows_of = [&](int bk, int64_t (&rr)[4]) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int e = bk * kBlk + static_cast<int>(rank) * kRows + 16 * gw + 4 * i + rsub;
          const int v = e < p.k ? __ldg(I.idx_row + e) : -1;
          rr[i] = (v >= 0 && v < I.len) ? cache_row(I, v) : -1;
        }
      };
      int64_t cur[4], nxt[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { cur[i] = -1; nxt[i] = -1; }
      if (nblk > 0) rows_of(blk0, cur);
      for (int j = 0; j < nblk && ok; ++j) {
        if (j + 1 < nblk) rows_of(blk0 + j + 1, nxt);
        const uint16_t* src[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) src[h] = p.kv + (cur[h] < 0 ? 0 : cur[h]) * DSA_D_QK + c16 * 8;
        for (int i = 0; i < kDChunks; ++i) {
          const int c = chunk_at(i);
          if (!warp_wait(&S.s_empty[slot], sph ^ 1, p.status, ab, false)) { ok = false; break; }
          const uint32_t dst0 = smem_u32(S.s_ring[slot]);
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const int r = 16 * gw + 4 * h + rsub;              // row within this CTA's 128
            cp_async16(dst0 + r * 128 + ((c16 ^ (r & 7)) << 4), src[h] + c * 64, cur[h] < 0 ? 0u : 16u);
          }
          cp_async_arrive_noinc(&S.s_loaded[slot]);
          if (++slot == kSStages) { slot = 0; sph ^= 1; }
        }
#pragma unroll
        for (int h = 0; h < 4; ++h) cur[h] = nxt[h];
      }
      if (ok && it + ncl < n_items) ok = scan(kk + 1, it + ncl);
    }
    cp_async_wait_all();
  } else if (warp < 4 + kSWarps + kVWarps) {
    // ================================================================ V gathers
    // Warps 12-19 gather the V operand straight from L2, slice by slice: a
    // slice is 32 rows of the block (both CTAs' rows) with this CTA's value
    // dims, dim group g (0..3) = dims (g/2)*256 + r*128 + (g%2)*64 (MN-major
    // SW128: one 128-byte line per row and group).  Warp w loads rows
    // 4w..4w+3 of every slice, one 16-byte copy per lane and row (lane =
    // group * 8 + chunk).  The block's indices are read once: lane l holds the
    // row 4w + (l & 3) of slice l >> 2.  A slot is refilled as soon as the PV
    // MMAs have read it.
    const int vw = warp - 4 - kSWarps;
    const int g = lane >> 3;
    const int c16 = lane & 7;
    const int dim0 = (g >> 1) * 256 + static_cast<int>(rank) * 128 + (g & 1) * 64 + c16 * 8;
    int slot = 0;
    uint32_t vph = 0;
    bool ok = true;
    for (int kk = 0, it = cid; it < n_items && ok; ++kk, it += ncl) {
      const int b = kk & 1;
      if (!warp_wait(&S.plan_ready[b], (kk >> 1) & 1, p.status, ab, false)) break;
      const Item I = item_of(it);
      int blk0, nblk;
      plan_of(b, I.split, blk0, nblk);
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.plan_free[b]);
      auto row_of = [&](int bk) -> int64_t {
        const int e = bk * kBlk + (lane >> 2) * kVRows + 4 * vw + (lane & 3);
        const int v = e < p.k ? __ldg(I.idx_row + e) : -1;
        return (v >= 0 && v < I.len) ? cache_row(I, v) : -1;
      };
      int64_t cur = nblk > 0 ? row_of(blk0) : -1, nxt = -1;
      for (int j = 0; j < nblk && ok; ++j) {
        if (j + 1 < nblk) nxt = row_of(blk0 + j + 1);
        for (int vs = 0; vs < kVSlices; ++vs) {
          if (!warp_wait(&S.v_empty[slot], vph ^ 1, p.status, ab, false)) { ok = false; break; }
          const uint32_t dst0 = smem_u32(S.v_ring[slot][g]);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int64_t v = __shfl_sync(0xffffffffu, cur, vs * 4 + i);
            const int r = 4 * vw + i;                          // row of the slice
            cp_async16(dst0 + r * 128 + ((c16 ^ (r & 7)) << 4),
                       p.kv + (v < 0 ? 0 : v) * DSA_D_QK + dim0, v < 0 ? 0u : 16u);
          }
          cp_async_arrive_noinc(&S.v_loaded[slot]);
          if (++slot == kVStages) { slot = 0; vph ^= 1; }
        }
        cur = nxt;
      }
    }
    cp_async_wait_all();
  } else if (warp == kRoleWarp && lane == 0) {
    // ================================================================ Q loads + S MMAs
    // In both CTAs: this CTA's Q of the next query (9 TMA boxes of 64 dims x 64
    // heads) once the S MMAs of the previous query have completed.  In the even
    // CTA it then issues S = Q K^T block after block.  Waits use the CTA-scope
    // try_wait, as 2-SM tensor-core pipelines do for the leader's stage
    // barriers.  Descriptors are built once; a step inside a tile adds to the
    // 14-bit start-address field (16-byte units).
    const uint32_t id_s = instr_desc(1, 1, false, false, 128, kBlk);   // bf16 x bf16, M=128 pair, N=256
    const uint64_t qd0 = smem_desc_sw128(smem_u32(S.q[0]), 16, 1024);
    const uint64_t sd0 = smem_desc_sw128(smem_u32(S.s_ring[0]), 16, 1024);
    int gb = 0, slot = 0;
    uint32_t sph = 0, nq = 0;
    bool ok = true;
    for (int kk = 0, it = cid; it < n_items && ok; ++kk, it += ncl) {
      const int b = kk & 1;
      if (!mbar_wait(&S.plan_ready[b], (kk >> 1) & 1, p.status, ab)) break;
      const Item I = item_of(it);
      int blk0, nblk;
      plan_of(b, I.split, blk0, nblk);
      mbar_arrive(&S.plan_free[b]);
      if (nblk == 0) continue;
      if (nq > 0 && !mbar_wait(&S.q_empty, (nq - 1) & 1, p.status, ab)) break;
      mbar_arrive_expect_tx(&S.q_full, kDChunks * kHeads * 128);
      for (int dc = 0; dc < kDChunks; ++dc)
        tma_load_2d(S.q[dc], &tm_q, &S.q_full, dc * 64, I.t * H + head0);
      if (!mbar_wait(&S.q_full, nq & 1, p.status, ab)) break;
      pair_signal(rank, &S.q_ready, &S.mbox_q, true, 4);
      if (rank == 0) {
        if (!mbar_wait(&S.q_ready, nq & 1, p.status, ab)) break;
        for (int j = 0; j < nblk && ok; ++j, ++gb) {
          const int sb = gb & 1;
          if (!mbar_wait(&S.s_free[sb], ((gb >> 1) & 1) ^ 1, p.status, ab)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d = tmem + kSCol + sb * 128;
          for (int ci = 0; ci < kDChunks; ++ci) {
            const int dc = chunk_at(ci);
            if (!mbar_wait(&S.s_full[slot], sph, p.status, ab)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int kk4 = 0; kk4 < 4; ++kk4)
              umma_bf16_pair(d, qd0 + static_cast<uint64_t>(dc * (kHeads * 128 / 16) + kk4 * 2),
                             sd0 + static_cast<uint64_t>(slot * (kRows * 128 / 16) + kk4 * 2), id_s,
                             (ci | kk4) != 0 ? 1u : 0u);
            umma_commit_pair(&S.s_empty[slot], 0x3);
            if (++slot == kSStages) { slot = 0; sph ^= 1; }
          }
          if (!ok) break;
          umma_commit_pair(&S.s_ready[sb], 0x3);
        }
        if (!ok) break;
        umma_commit_pair(&S.q_empty, 0x3);                 // Q is free once these MMAs completed
      }
      ++nq;
    }
    if (rank == 0) {
      umma_commit_pair(&S.done, 0x1);                     // drain: this issuer's MMAs completed
      mbar_wait(&S.done, 0, p.status, nullptr);            // ... and the other issuer's
    }
  } else if (warp == kRoleWarp + 1 && lane == 0) {
    // ================================================================ S relay
    // Forwards completed S-ring stages, in order, to the even CTA's barriers.
    // It waits with the suspending try_wait: a spinning test_wait poller
    // competes with the gathers for the shared-memory pipe.
    int slot = 0;
    uint32_t sph = 0;
    bool ok = true;
    for (int kk = 0, it = cid; it < n_items && ok; ++kk, it += ncl) {
      const int b = kk & 1;
      if (!mbar_wait(&S.plan_ready[b], (kk >> 1) & 1, p.status, ab)) break;
      const Item I = item_of(it);
      int blk0, nblk;
      plan_of(b, I.split, blk0, nblk);
      mbar_arrive(&S.plan_free[b]);
      for (int gi = 0; gi < nblk * kDChunks; ++gi) {
        if (!mbar_wait(&S.s_loaded[slot], sph, p.status, ab)) { ok = false; break; }
        fence_proxy_async_smem();                          // cp.async writes -> tensor-core reads
        pair_signal(rank, &S.s_full[slot], &S.mbox_s[slot], true, 4);
        if (++slot == kSStages) { slot = 0; sph ^= 1; }
      }
    }
  } else if (warp == kRoleWarp + 2 && lane == 0) {
    // ================================================================ V relay
    // Forwards each landed V slice of this CTA to the even CTA's v_full barrier,
    // which the PV issuer waits on.
    int slot = 0;
    uint32_t vph = 0;
    bool ok = true;
    for (int kk = 0, it = cid; it < n_items && ok; ++kk, it += ncl) {
      const int b = kk & 1;
      if (!mbar_wait(&S.plan_ready[b], (kk >> 1) & 1, p.status, ab)) break;
      const Item I = item_of(it);
      int blk0, nblk;
      plan_of(b, I.split, blk0, nblk);
      mbar_arrive(&S.plan_free[b]);
      for (int gv = 0; gv < nblk * kVSlices; ++gv) {
        if (!mbar_wait(&S.v_loaded[slot], vph, p.status, ab)) { ok = false; break; }
        fence_proxy_async_smem();                          // cp.async writes -> tensor-core reads
        pair_signal(rank, &S.v_full[slot], &S.mbox_v[slot], true, 4);
        if (++slot == kVStages) { slot = 0; vph ^= 1; }
      }
    }
  } else if (warp == kRoleWarp + 3 && lane == 0 && rank == 0) {
    // ================================================================ PV MMAs (even CTA)
    // O += P V, slice by slice; the tensor pipe executes the S and PV streams,
    // which touch disjoint TMEM columns.  The first PV of a query overwrites O,
    // so it waits until both CTAs have read the previous query's O out.
    const uint32_t id_pv = instr_desc(1, 1, false, true, 128, 256);    // B (V) MN-major, N=256
    const uint64_t pd0 = smem_desc_sw128(smem_u32(S.p[0]), 16, 1024);
    const uint64_t vd0 = smem_desc_sw128(smem_u32(S.v_ring[0][0]), kVRows * 128, 1024);
    int gb = 0, slot = 0;
    uint32_t vph = 0, ne = 0;
    bool ok = true;
    for (int kk = 0, it = cid; it < n_items && ok; ++kk, it += ncl) {
      const int b = kk & 1;
      if (!mbar_wait(&S.plan_ready[b], (kk >> 1) & 1, p.status, ab)) break;
      const Item I = item_of(it);
      int blk0, nblk;
      plan_of(b, I.split, blk0, nblk);
      mbar_arrive(&S.plan_free[b]);
      if (nblk == 0) continue;
      if (ne > 0 && !mbar_wait(&S.o_free, (ne - 1) & 1, p.status, ab)) break;
      for (int j = 0; j < nblk && ok; ++j, ++gb) {
        if (!mbar_wait(&S.p_full[0], gb & 1, p.status, ab)) { ok = false; break; }
        tc_fence_after();
        // slice by slice: each V slot's four MMAs (two 16-row K steps x two
        // halves of the value dims) release it for the gathers of a later slice
        for (int vs = 0; vs < kVSlices; ++vs) {
          if (vs == kVSlices / 2) {
            // rows 0..127 of P consumed: half 0 of the next block may overwrite
            // them; rows 128..255 must have been written by now
            umma_commit_pair(&S.p_empty[0], 0x3);
            if (!mbar_wait(&S.p_full[1], gb & 1, p.status, ab)) { ok = false; break; }
            tc_fence_after();
          }
          if (!mbar_wait(&S.v_full[slot], vph, p.status, ab)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int k2 = 0; k2 < 2; ++k2) {
            const int ks = vs * 2 + k2;                      // 16-row K step of the block
            const uint64_t pa = pd0 + static_cast<uint64_t>((ks >> 2) * (kHeads * 128 / 16) + (ks & 3) * 2);
#pragma unroll
            for (int c = 0; c < 2; ++c)
              umma_bf16_pair(tmem + kOCol + c * 128, pa,
                             vd0 + static_cast<uint64_t>(slot * (4 * kVRows * 128 / 16) + c * (2 * kVRows * 128 / 16) +
                                                         k2 * (16 * 128 / 16)),
                             id_pv, (j | ks) != 0 ? 1u : 0u);
          }
          umma_commit_pair(&S.v_empty[slot], 0x3);
          if (++slot == kVStages) { slot = 0; vph ^= 1; }
        }
        if (!ok) break;
        umma_commit_pair(&S.p_empty[1], 0x3);
      }
      if (!ok) break;
      umma_commit_pair(&S.o_full, 0x3);                   // O of this query is complete once these MMAs are
      ++ne;
    }
    umma_commit_pair(&S.done, 0x1);                       // drain: this issuer's MMAs completed
    mbar_wait(&S.done, 0, p.status, nullptr);              // ... and the other issuer's
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  if (warp == kRoleWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// Merge split partial results: lse = log sum exp(lse_i); out = sum exp(lse_i - lse) o_i.
__global__ void __launch_bounds__(128) mla_combine_kernel(MlaParams p) {
  const int t = blockIdx.x, h = blockIdx.y;
  const int64_t pr = (static_cast<int64_t>(t) * p.splits) * p.H + h;
  float mx = -INFINITY;
  for (int s = 0; s < p.splits; ++s) mx = fmaxf(mx, p.part_lse[pr + static_cast<int64_t>(s) * p.H]);
  float den = 0.f;
  for (int s = 0; s < p.splits; ++s) {
    const float ls = p.part_lse[pr + static_cast<int64_t>(s) * p.H];
    den += ls == -INFINITY ? 0.f : __expf(ls - mx);
  }
  const int d = threadIdx.x * 4;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < p.splits; ++s) {
    const float ls = p.part_lse[pr + static_cast<int64_t>(s) * p.H];
    if (ls == -INFINITY) continue;
    const float wgt = __expf(ls - mx) / den;
    const float4 o = *reinterpret_cast<const float4*>(p.part_o + (pr + static_cast<int64_t>(s) * p.H) * DSA_D_V + d);
    acc.x += wgt * o.x; acc.y += wgt * o.y; acc.z += wgt * o.z; acc.w += wgt * o.w;
  }
  uint16_t* orow = p.out + (static_cast<int64_t>(t) * p.H + h) * DSA_D_V + d;
  *reinterpret_cast<uint2*>(orow) = make_uint2(pack_bf16(acc.x, acc.y), pack_bf16(acc.z, acc.w));
  if (threadIdx.x == 0 && p.lse)
    p.lse[static_cast<int64_t>(t) * p.H + h] = den > 0.f ? mx + __logf(den) : -INFINITY;
}

}  // namespace

static_assert(sizeof(MlaSmem) <= 232448, "sparse-MLA shared memory exceeds the 227 KB per-CTA limit");

size_t mla_smem_bytes() { return sizeof(MlaSmem); }

cudaError_t launch_sparse_mla(const MlaParams& p, const CUtensorMap& tm_q, cudaStream_t stream) {
  if (p.T == 0) return cudaSuccess;
  const size_t smem = mla_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(sparse_mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  // The in-kernel register split adds up to the launch allocation only at
  // kLaunchRegs per thread; with fewer, the softmax warpgroup's increase could
  // never be granted.  Refuse to launch rather than wait forever.
  static int regs = -1;
  if (regs < 0) {
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, sparse_mla_kernel);
    if (e != cudaSuccess) return e;
    regs = fa.numRegs;
  }
  if (regs != static_cast<int>(kLaunchRegs)) return cudaErrorInvalidConfiguration;
  // persistent pairs: as many as can be resident at once, at most one per item
  static int max_pairs = -1;
  if (max_pairs < 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(kMlaThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, sparse_mla_kernel, &cfg) != cudaSuccess || n <= 0) {
      (void)cudaGetLastError();
      int dev = 0, sms = 0;
      if (cudaGetDevice(&dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 2)
        sms = 2;
      n = sms / 2;
    }
    max_pairs = n;
  }
  const int64_t items = static_cast<int64_t>(p.T) * p.splits;
  const int pairs = static_cast<int>(items < max_pairs ? items : max_pairs);
  sparse_mla_kernel<<<2 * pairs, kMlaThreads, smem, stream>>>(tm_q, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  count_launches(1);
  if (p.splits == 1) return e;
  mla_combine_kernel<<<dim3(p.T, p.H), 128, 0, stream>>>(p);
  e = cudaGetLastError();
  if (e == cudaSuccess) count_launches(1);
  return e;
}

}  // namespace dsa
