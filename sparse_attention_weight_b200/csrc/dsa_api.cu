// C ABI of the DSA hot path (declared in include/dsa.h): argument checks,
// workspace layout, TMA descriptors and launches on the caller's stream.
#include <atomic>
#include <cstring>
#include <mutex>

#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {

static std::atomic<uint64_t> g_launches{0};
void count_launches(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D row-major tensor [rows, cols] of `elem` bytes, 128-byte swizzled boxes.
bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, size_t elem, const void* base, uint64_t cols,
                 uint64_t rows, uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * elem};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool batch_ok(const dsa_batch* b) {
  if (!b) return false;
  if (b->num_seqs < 1 || b->num_q < 0 || b->max_kv_len < 1 || b->max_q_per_seq < 0 || b->kv_rows < 0) return false;
  if (b->page_size < 0 || b->pages_per_seq < 0) return false;
  if (b->num_q > 0) {
    if (!b->kv_len || !b->q_seq || !b->q_pos) return false;
    if (b->page_size == 0 ? !b->kv_offset : !b->page_table) return false;
  }
  if (b->page_size > 0 && static_cast<int64_t>(b->pages_per_seq) * b->page_size < b->max_kv_len) return false;
  return true;
}

// Paged caches: pages of a multiple of 64 rows (the indexer loads 64-key halves
// of its 128-key tiles, each from one page), whole pages of physical rows.
bool paging_ok(const dsa_batch* b) {
  return b->page_size == 0 || (b->page_size % 64 == 0 && b->kv_rows % b->page_size == 0);
}

bool hi_ok(int H_I) { return H_I >= 4 && H_I <= 64 && H_I % 4 == 0; }
// Column stride of one query token in the indexer's MMA: H_I rounded up to a
// power of two (the epilogue reads whole 32-column TMEM chunks per token).
int hi_pad(int H_I) {
  int p = 4;
  while (p < H_I) p <<= 1;
  return p;
}
bool h_ok(int H) { return H >= 8 && H <= 128 && H % 8 == 0; }
// The indexer emits per-row key histograms when its query groups hold at most
// four tokens (one shared-memory histogram per token slot) of >= 32 padded heads.
int indexer_group(const dsa_batch* b, int H_I);
bool hist_supported(const dsa_batch* b, int H_I) { return hi_pad(H_I) >= 32 && indexer_group(b, H_I) <= 4; }
bool k_ok(int k) { return k >= 1 && k <= 2048; }

int64_t default_ld(const dsa_batch* b) { return (static_cast<int64_t>(b->max_kv_len) + 3) / 4 * 4; }

// Query tokens per indexer group: a power of two covering the queries of one
// sequence, with the MMA N = G * hi_pad(H_I) in [16, 256].
int indexer_group(const dsa_batch* b, int H_I) {
  const int hp = hi_pad(H_I);
  int want = b->max_q_per_seq > 0 ? b->max_q_per_seq : b->num_q;
  int g = 1;
  while (g < want && g * hp < 256) g <<= 1;
  while (g * hp < 16) g <<= 1;
  return g;
}

// Splits of each query's index list in the sparse-MLA kernel: enough CTA pairs
// to fill one wave of the SMs when there are few queries.
int mla_splits(const dsa_batch* b, int k) {
  const int pairs = num_sms() / 2;
  const int blocks = (k + 255) / 256;            // the kernel walks an index row in blocks of 256
  if (b->num_q <= 0) return 1;
  int s = pairs / b->num_q;
  if (s < 1) s = 1;
  if (s > blocks) s = blocks;
  if (s > 16) s = 16;
  return s;
}

int proj_rows(int H_I, int H) { return H_I * DSA_D_INDEX + DSA_D_INDEX + H_I + DSA_D_QK + H * DSA_D_QK; }

size_t plan_bytes(const dsa_batch* b) { return align_up((6 * static_cast<size_t>(b->num_q) + 2) * sizeof(int32_t)); }

struct WsLayout {
  uint32_t* status;
  int32_t* plan;
  float* part_o;
  float* part_lse;
  float* scores;
  int32_t* idx;
  size_t bytes;
};

struct ProjLayout {
  uint32_t* status;
  float* y;
  void* gemm_ws;
  size_t bytes;
};

ProjLayout proj_layout(void* ws, const dsa_batch* b, int H_I, int H) {
  ProjLayout L{};
  uint8_t* p = static_cast<uint8_t*>(ws);
  size_t off = kWsHeader;
  L.status = reinterpret_cast<uint32_t*>(p);
  L.y = reinterpret_cast<float*>(p + off);
  off += align_up(static_cast<size_t>(b->num_q) * proj_rows(H_I, H) * sizeof(float));
  L.gemm_ws = p + off;
  off += project_gemm_workspace_bytes();
  L.bytes = off;
  return L;
}

WsLayout layout(void* ws, int op, const dsa_batch* b, int H, int k, int64_t ld) {
  WsLayout L{};
  uint8_t* p = static_cast<uint8_t*>(ws);
  size_t off = kWsHeader;
  L.status = reinterpret_cast<uint32_t*>(p);
  if (op == DSA_OP_INDEXER || op == DSA_OP_FORWARD) {
    L.plan = reinterpret_cast<int32_t*>(p + off);
    off += plan_bytes(b);
  }
  if (op == DSA_OP_SPARSE_MLA || op == DSA_OP_FORWARD) {
    const int s = mla_splits(b, k);
    if (s > 1) {
      const size_t rows = static_cast<size_t>(b->num_q) * s * H;
      L.part_o = reinterpret_cast<float*>(p + off);
      off += align_up(rows * DSA_D_V * sizeof(float));
      L.part_lse = reinterpret_cast<float*>(p + off);
      off += align_up(rows * sizeof(float));
    }
  }
  if (op == DSA_OP_FORWARD) {
    L.scores = reinterpret_cast<float*>(p + off);
    off += align_up(static_cast<size_t>(b->num_q) * ld * sizeof(float));
    L.idx = reinterpret_cast<int32_t*>(p + off);
    off += align_up(static_cast<size_t>(b->num_q) * k * sizeof(int32_t));
  }
  L.bytes = off;
  return L;
}

dsa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA; }

// dsa_forward_host: about sixteen query chunks of at least 256 queries (so a chunk
// fills the sparse-MLA kernel's pairs without split-KV when T is large).
constexpr int kHostChunks = 16;
constexpr int kHostMinChunk = 256;
int host_chunk(int T) {
  const int c = (T + kHostChunks - 1) / kHostChunks;
  return c < kHostMinChunk ? kHostMinChunk : c;
}
// The queries [q0, q0 + n) of a batch, against the same cache.
dsa_batch chunk_batch(const dsa_batch* b, int q0, int n) {
  dsa_batch s = *b;
  s.num_q = n;
  s.q_seq = b->q_seq + q0;
  s.q_pos = b->q_pos + q0;
  return s;
}
// The largest forward workspace of the chunks (a short last chunk may need the
// split-KV partials that the full-size chunks do not).
size_t host_ws_bytes(const dsa_batch* b, int H, int k) {
  const int T = b->num_q, c = host_chunk(T);
  size_t m = kWsHeader;
  for (int q0 = 0; q0 < T; q0 += c) {
    const dsa_batch s = chunk_batch(b, q0, T - q0 < c ? T - q0 : c);
    const size_t n = layout(nullptr, DSA_OP_FORWARD, &s, H, k, default_ld(b)).bytes;
    if (n > m) m = n;
  }
  return m;
}
bool pinned_host(const void* p) {
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeHost;
}
// Events of one call, destroyed on every return path (a recorded event is
// released by the driver once it completes).
struct EventSet {
  cudaEvent_t e[4 + 2 * (kHostChunks + 1)];
  int n = 0;
  cudaEvent_t make() {
    if (n == static_cast<int>(sizeof(e) / sizeof(e[0]))) return nullptr;
    cudaEvent_t x = nullptr;
    if (cudaEventCreateWithFlags(&x, cudaEventDisableTiming) != cudaSuccess) return nullptr;
    e[n++] = x;
    return x;
  }
  ~EventSet() {
    for (int i = 0; i < n; ++i) cudaEventDestroy(e[i]);
  }
};
// `to` waits for the work queued so far on `from`.
bool order_after(EventSet& E, cudaStream_t from, cudaStream_t to) {
  cudaEvent_t x = E.make();
  return x && cudaEventRecord(x, from) == cudaSuccess && cudaStreamWaitEvent(to, x, 0) == cudaSuccess;
}

dsa_status run_indexer(const dsa_batch* b, const uint8_t* q_idx, const uint8_t* k_idx, const float* w, int H_I,
                       float* scores, int64_t ld, const WsLayout& L, cudaStream_t st, uint32_t* hist = nullptr) {
  if (b->num_q == 0) return DSA_OK;
  const int G = indexer_group(b, H_I);
  const int hp = hi_pad(H_I);
  CUtensorMap tq, tk;
  // one box per query group, or (H_I not a power of two) one box per token
  if (!make_map_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q_idx, DSA_D_INDEX,
                   static_cast<uint64_t>(b->num_q) * H_I, DSA_D_INDEX,
                   static_cast<uint32_t>(hp == H_I ? G * H_I : H_I)))
    return DSA_ERR_CUDA;
  if (!make_map_2d(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, k_idx, DSA_D_INDEX,
                   static_cast<uint64_t>(b->kv_rows > 0 ? b->kv_rows : 1), DSA_D_INDEX, 64))
    return DSA_ERR_CUDA;
  const int T = b->num_q;
  IndexerParams p{};
  p.w = w;
  p.scores = scores;
  p.ld = ld;
  p.q_seq = b->q_seq;
  p.q_pos = b->q_pos;
  p.kv_offset = b->kv_offset;
  p.kv_len = b->kv_len;
  p.page_table = b->page_table;
  p.page_size = b->page_size;
  p.pages_per_seq = b->pages_per_seq;
  p.kv_rows = b->kv_rows;
  p.hist = hist;
  int32_t* plan = L.plan;
  p.group_q0 = plan;
  p.group_cnt = plan + T;
  p.group_seq = plan + 2 * T;
  p.group_tiles = plan + 3 * T;
  p.item_off = plan + 4 * T;           // T + 1 entries
  p.ngroups = plan + 5 * T + 1;
  p.q_nvis = plan + 5 * T + 2;         // T entries (plan has 6T + 2)
  p.status = L.status;
  p.G = G;
  p.hi = H_I;
  p.nacc = G * hp <= 128 ? 4 : 2;
  p.max_kv_len = b->max_kv_len;
  return cuda_status(launch_indexer(tq, tk, p, hp, T, b->num_seqs, b->kv_rows, num_sms(), st));
}

dsa_status run_topk(const dsa_batch* b, const float* scores, int64_t ld, int k, int32_t* idx, const WsLayout& L,
                    cudaStream_t st, const uint32_t* hist = nullptr) {
  TopkParams p{};
  p.scores = scores;
  p.hist = hist;
  p.ld = ld;
  p.idx = idx;
  p.k = k;
  p.q_seq = b->q_seq;
  p.q_pos = b->q_pos;
  p.kv_len = b->kv_len;
  p.num_seqs = b->num_seqs;
  p.max_kv_len = b->max_kv_len;
  p.status = L.status;
  return cuda_status(launch_topk(p, b->num_q, st));
}

dsa_status run_mla(const dsa_batch* b, const uint16_t* q, const uint16_t* kv, const int32_t* idx, int k, int H,
                   float sm_scale, uint16_t* out, float* lse, const WsLayout& L, cudaStream_t st) {
  if (b->num_q == 0) return DSA_OK;
  CUtensorMap tq;
  if (!make_map_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q, DSA_D_QK, static_cast<uint64_t>(b->num_q) * H, 64,
                   64))
    return DSA_ERR_CUDA;
  MlaParams p{};
  p.q = q;
  p.kv = kv;
  p.idx = idx;
  p.k = k;
  p.H = H;
  p.sm_scale = sm_scale;
  p.sm_scale_log2 = sm_scale * 1.4426950408889634f;
  p.out = out;
  p.lse = lse;
  p.q_seq = b->q_seq;
  p.q_pos = b->q_pos;
  p.kv_offset = b->kv_offset;
  p.kv_len = b->kv_len;
  p.page_table = b->page_table;
  p.page_size = b->page_size;
  p.pages_per_seq = b->pages_per_seq;
  p.num_seqs = b->num_seqs;
  p.kv_rows = b->kv_rows;
  p.T = b->num_q;
  p.splits = mla_splits(b, k);
  p.part_o = L.part_o;
  p.part_lse = L.part_lse;
  p.status = L.status;
  return cuda_status(launch_sparse_mla(p, tq, st));
}

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" {

size_t dsa_workspace_size(int op, const dsa_batch* batch, int H_I, int H, int k, int64_t ld) {
  if (!batch_ok(batch)) return 0;
  if (op == DSA_OP_PROJECT) return hi_ok(H_I) && h_ok(H) ? proj_layout(nullptr, batch, H_I, H).bytes : 0;
  if (op == DSA_OP_MLA_BACKWARD) return kWsHeader;
  if (op == DSA_OP_FORWARD_HOST) return hi_ok(H_I) && h_ok(H) && k_ok(k) ? host_ws_bytes(batch, H, k) : 0;
  if (op < DSA_OP_INDEXER || op > DSA_OP_FORWARD) return 0;
  if ((op == DSA_OP_SPARSE_MLA || op == DSA_OP_FORWARD) && (!h_ok(H) || !k_ok(k))) return 0;
  if (op == DSA_OP_FORWARD && !k_ok(k)) return 0;
  if (ld <= 0) ld = default_ld(batch);
  return layout(nullptr, op, batch, H, k, ld).bytes;
}

dsa_status dsa_indexer_scores(const dsa_batch* batch, const uint8_t* q_idx, const uint8_t* k_idx, const float* w,
                              int H_I, float* scores, int64_t ld, void* ws, size_t ws_bytes, void* stream) {
  if (!batch_ok(batch) || !ws) return DSA_ERR_INVALID_ARGUMENT;
  if (batch->num_q > 0 && (!q_idx || !k_idx || !w || !scores)) return DSA_ERR_INVALID_ARGUMENT;
  if (!hi_ok(H_I) || !paging_ok(batch)) return DSA_ERR_UNSUPPORTED;
  if (ld < batch->max_kv_len || ld % 4 != 0) return DSA_ERR_UNSUPPORTED;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(w) || !aligned16(scores) || !aligned16(ws))
    return DSA_ERR_UNSUPPORTED;
  const WsLayout L = layout(ws, DSA_OP_INDEXER, batch, 8, 1, ld);
  if (ws_bytes < L.bytes) return DSA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(L.status, 0, sizeof(uint32_t), st) != cudaSuccess) return DSA_ERR_CUDA;
  return run_indexer(batch, q_idx, k_idx, w, H_I, scores, ld, L, st);
}

dsa_status dsa_topk(const dsa_batch* batch, const float* scores, int64_t ld, int k, int32_t* idx, void* ws,
                    size_t ws_bytes, void* stream) {
  if (!batch_ok(batch) || !ws) return DSA_ERR_INVALID_ARGUMENT;
  if (batch->num_q > 0 && (!scores || !idx)) return DSA_ERR_INVALID_ARGUMENT;
  if (!k_ok(k)) return DSA_ERR_UNSUPPORTED;
  if (ld < batch->max_kv_len || ld % 4 != 0) return DSA_ERR_UNSUPPORTED;
  if (!aligned16(scores) || !aligned16(ws)) return DSA_ERR_UNSUPPORTED;
  const WsLayout L = layout(ws, DSA_OP_TOPK, batch, 8, k, ld);
  if (ws_bytes < L.bytes) return DSA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(L.status, 0, sizeof(uint32_t), st) != cudaSuccess) return DSA_ERR_CUDA;
  return run_topk(batch, scores, ld, k, idx, L, st);
}

dsa_status dsa_indexer_scores_hist(const dsa_batch* batch, const uint8_t* q_idx, const uint8_t* k_idx, const float* w,
                                   int H_I, float* scores, int64_t ld, uint32_t* hist, void* ws, size_t ws_bytes,
                                   void* stream) {
  if (!batch_ok(batch) || !ws) return DSA_ERR_INVALID_ARGUMENT;
  if (batch->num_q > 0 && (!q_idx || !k_idx || !w || !scores || !hist)) return DSA_ERR_INVALID_ARGUMENT;
  if (!hi_ok(H_I) || !paging_ok(batch) || !hist_supported(batch, H_I)) return DSA_ERR_UNSUPPORTED;
  if (ld < batch->max_kv_len || ld % 4 != 0) return DSA_ERR_UNSUPPORTED;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(w) || !aligned16(scores) || !aligned16(hist) ||
      !aligned16(ws))
    return DSA_ERR_UNSUPPORTED;
  const WsLayout L = layout(ws, DSA_OP_INDEXER, batch, 8, 1, ld);
  if (ws_bytes < L.bytes) return DSA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(L.status, 0, sizeof(uint32_t), st) != cudaSuccess) return DSA_ERR_CUDA;
  if (batch->num_q > 0 &&
      cudaMemsetAsync(hist, 0, static_cast<size_t>(batch->num_q) * 2048 * sizeof(uint32_t), st) != cudaSuccess)
    return DSA_ERR_CUDA;
  return run_indexer(batch, q_idx, k_idx, w, H_I, scores, ld, L, st, hist);
}

dsa_status dsa_topk_hist(const dsa_batch* batch, const float* scores, int64_t ld, const uint32_t* hist, int k,
                         int32_t* idx, void* ws, size_t ws_bytes, void* stream) {
  if (!batch_ok(batch) || !ws) return DSA_ERR_INVALID_ARGUMENT;
  if (batch->num_q > 0 && (!scores || !idx || !hist)) return DSA_ERR_INVALID_ARGUMENT;
  if (!k_ok(k)) return DSA_ERR_UNSUPPORTED;
  if (ld < batch->max_kv_len || ld % 4 != 0) return DSA_ERR_UNSUPPORTED;
  if (!aligned16(scores) || !aligned16(hist) || !aligned16(ws)) return DSA_ERR_UNSUPPORTED;
  const WsLayout L = layout(ws, DSA_OP_TOPK, batch, 8, k, ld);
  if (ws_bytes < L.bytes) return DSA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(L.status, 0, sizeof(uint32_t), st) != cudaSuccess) return DSA_ERR_CUDA;
  return run_topk(batch, scores, ld, k, idx, L, st, hist);
}

dsa_status dsa_sparse_mla_backward(const dsa_batch* batch, const uint16_t* q, const uint16_t* kv, const int32_t* idx,
                                   int k, int H, float sm_scale, const uint16_t* out, const float* lse,
                                   const uint16_t* d_out, float* d_q, float* d_kv, void* ws, size_t ws_bytes,
                                   void* stream) {
  if (!batch_ok(batch) || !ws) return DSA_ERR_INVALID_ARGUMENT;
  if (batch->num_q > 0 && (!q || !kv || !idx || !out || !lse || !d_out || !d_q || !d_kv))
    return DSA_ERR_INVALID_ARGUMENT;
  if (!h_ok(H) || !k_ok(k) || !paging_ok(batch)) return DSA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(kv) || !aligned16(out) || !aligned16(d_out) || !aligned16(d_q) ||
      !aligned16(d_kv) || !aligned16(ws))
    return DSA_ERR_UNSUPPORTED;
  if (ws_bytes < kWsHeader) return DSA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* status = static_cast<uint32_t*>(ws);
  if (cudaMemsetAsync(status, 0, sizeof(uint32_t), st) != cudaSuccess) return DSA_ERR_CUDA;
  MlaBwdParams p{};
  p.q = q;
  p.kv = kv;
  p.idx = idx;
  p.k = k;
  p.H = H;
  p.sm_scale = sm_scale;
  p.out = out;
  p.lse = lse;
  p.d_out = d_out;
  p.d_q = d_q;
  p.d_kv = d_kv;
  p.q_seq = batch->q_seq;
  p.kv_offset = batch->kv_offset;
  p.kv_len = batch->kv_len;
  p.page_table = batch->page_table;
  p.page_size = batch->page_size;
  p.pages_per_seq = batch->pages_per_seq;
  p.num_seqs = batch->num_seqs;
  p.kv_rows = batch->kv_rows;
  p.T = batch->num_q;
  p.status = status;
  return cuda_status(launch_mla_backward(p, st));
}

int dsa_topk_uses_hist(const dsa_batch* batch, int k) {
  if (!batch_ok(batch) || !k_ok(k)) return 0;
  return topk_uses_hist(batch->max_kv_len, batch->num_q, num_sms()) ? 1 : 0;
}

dsa_status dsa_sparse_mla(const dsa_batch* batch, const uint16_t* q, const uint16_t* kv, const int32_t* idx, int k,
                          int H, float sm_scale, uint16_t* out, float* lse, void* ws, size_t ws_bytes,
                          void* stream) {
  if (!batch_ok(batch) || !ws) return DSA_ERR_INVALID_ARGUMENT;
  if (batch->num_q > 0 && (!q || !kv || !idx || !out)) return DSA_ERR_INVALID_ARGUMENT;
  if (!h_ok(H) || !k_ok(k) || !paging_ok(batch)) return DSA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(kv) || !aligned16(out) || !aligned16(ws)) return DSA_ERR_UNSUPPORTED;
  const WsLayout L = layout(ws, DSA_OP_SPARSE_MLA, batch, H, k, 0);
  if (ws_bytes < L.bytes) return DSA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(L.status, 0, sizeof(uint32_t), st) != cudaSuccess) return DSA_ERR_CUDA;
  return run_mla(batch, q, kv, idx, k, H, sm_scale, out, lse, L, st);
}

dsa_status dsa_forward(const dsa_batch* batch, const uint8_t* q_idx, const uint8_t* k_idx, const float* w, int H_I,
                       const uint16_t* q, const uint16_t* kv, int H, int k, float sm_scale, uint16_t* out, float* lse,
                       void* ws, size_t ws_bytes, void* stream) {
  if (!batch_ok(batch) || !ws) return DSA_ERR_INVALID_ARGUMENT;
  if (batch->num_q > 0 && (!q_idx || !k_idx || !w || !q || !kv || !out)) return DSA_ERR_INVALID_ARGUMENT;
  if (!hi_ok(H_I) || !h_ok(H) || !k_ok(k) || !paging_ok(batch)) return DSA_ERR_UNSUPPORTED;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(w) || !aligned16(q) || !aligned16(kv) ||
      !aligned16(out) || !aligned16(ws))
    return DSA_ERR_UNSUPPORTED;
  const int64_t ld = default_ld(batch);
  const WsLayout L = layout(ws, DSA_OP_FORWARD, batch, H, k, ld);
  if (ws_bytes < L.bytes) return DSA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(L.status, 0, sizeof(uint32_t), st) != cudaSuccess) return DSA_ERR_CUDA;
  // The unfused indexer -> top-k: emitting the key histograms costs the
  // indexer's epilogue more than skipping the first pass saves the top-k, which
  // already reads each row once (measured; see dsa_indexer_scores_hist).
  dsa_status s = run_indexer(batch, q_idx, k_idx, w, H_I, L.scores, ld, L, st);
  if (s != DSA_OK) return s;
  s = run_topk(batch, L.scores, ld, k, L.idx, L, st);
  if (s != DSA_OK) return s;
  return run_mla(batch, q, kv, L.idx, k, H, sm_scale, out, lse, L, st);
}

dsa_status dsa_project_append(const dsa_batch* batch, const uint16_t* hidden, const uint16_t* w_all, int d_model,
                              int H_I, int H, float rope_base, uint8_t* q_idx, float* w, uint16_t* q,
                              uint8_t* k_idx, uint16_t* kv, void* ws, size_t ws_bytes, void* stream) {
  if (!batch_ok(batch) || !ws) return DSA_ERR_INVALID_ARGUMENT;
  if (batch->num_q > 0 && (!hidden || !w_all || !q_idx || !w || !q || !k_idx || !kv))
    return DSA_ERR_INVALID_ARGUMENT;
  if (d_model <= 0 || !(rope_base > 0.f)) return DSA_ERR_INVALID_ARGUMENT;
  if (!hi_ok(H_I) || !h_ok(H) || d_model % 8 != 0 || !paging_ok(batch)) return DSA_ERR_UNSUPPORTED;
  if (!aligned16(hidden) || !aligned16(w_all) || !aligned16(q_idx) || !aligned16(w) || !aligned16(q) ||
      !aligned16(k_idx) || !aligned16(kv) || !aligned16(ws))
    return DSA_ERR_UNSUPPORTED;
  const ProjLayout L = proj_layout(ws, batch, H_I, H);
  if (ws_bytes < L.bytes) return DSA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(L.status, 0, sizeof(uint32_t), st) != cudaSuccess) return DSA_ERR_CUDA;
  if (batch->num_q == 0) return DSA_OK;
  ProjParams p{};
  p.y = L.y;
  p.q_idx = q_idx;
  p.w = w;
  p.q = q;
  p.k_cache = k_idx;
  p.kv_cache = kv;
  p.q_seq = batch->q_seq;
  p.q_pos = batch->q_pos;
  p.kv_offset = batch->kv_offset;
  p.kv_len = batch->kv_len;
  p.page_table = batch->page_table;
  p.page_size = batch->page_size;
  p.pages_per_seq = batch->pages_per_seq;
  p.num_seqs = batch->num_seqs;
  p.kv_rows = batch->kv_rows;
  p.T = batch->num_q;
  p.n_all = proj_rows(H_I, H);
  p.hi = H_I;
  p.heads = H;
  p.rope_base = rope_base;
  p.status = L.status;
  bool gemm_failed = false;
  const cudaError_t e = launch_project(p, hidden, w_all, d_model, L.gemm_ws, project_gemm_workspace_bytes(), st,
                                       &gemm_failed);
  return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status dsa_forward_host(const dsa_batch* batch, const uint8_t* h_q_idx, const float* h_w, const uint16_t* h_q,
                            const uint8_t* h_k_idx, const uint16_t* h_kv, uint8_t* q_idx, float* w, uint16_t* q,
                            uint8_t* k_idx, uint16_t* kv, int H_I, int H, int k, float sm_scale, uint16_t* out,
                            float* lse, uint16_t* h_out, void* ws, size_t ws_bytes, void* const streams[3]) {
  if (!batch_ok(batch) || !ws || !streams) return DSA_ERR_INVALID_ARGUMENT;
  const int T = batch->num_q;
  if (T > 0 && (!h_q_idx || !h_w || !h_q || !h_k_idx || !h_kv || !q_idx || !w || !q || !k_idx || !kv || !out ||
                !h_out))
    return DSA_ERR_INVALID_ARGUMENT;
  if (!hi_ok(H_I) || !h_ok(H) || !k_ok(k) || !paging_ok(batch)) return DSA_ERR_UNSUPPORTED;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(w) || !aligned16(q) || !aligned16(kv) ||
      !aligned16(out) || !aligned16(ws))
    return DSA_ERR_UNSUPPORTED;
  if (ws_bytes < host_ws_bytes(batch, H, k)) return DSA_ERR_WORKSPACE_TOO_SMALL;
  if (T > 0 && (!pinned_host(h_q_idx) || !pinned_host(h_w) || !pinned_host(h_q) || !pinned_host(h_k_idx) ||
                !pinned_host(h_kv) || !pinned_host(h_out)))
    return DSA_ERR_UNSUPPORTED;
  cudaStream_t s_in = static_cast<cudaStream_t>(streams[0]);
  cudaStream_t s_cp = static_cast<cudaStream_t>(streams[1]);
  cudaStream_t s_out = static_cast<cudaStream_t>(streams[2]);
  EventSet E;
  // after the earlier copies out of `out`, then the earlier readers of the inputs
  if (!order_after(E, s_out, s_cp) || !order_after(E, s_cp, s_in)) return DSA_ERR_CUDA;
  if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), s_cp) != cudaSuccess) return DSA_ERR_CUDA;
  if (T == 0) return DSA_OK;
  const size_t rows = static_cast<size_t>(batch->kv_rows);
  if (cudaMemcpyAsync(k_idx, h_k_idx, rows * DSA_D_INDEX, cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
      cudaMemcpyAsync(kv, h_kv, rows * DSA_D_QK * 2, cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
      !order_after(E, s_in, s_cp))
    return DSA_ERR_CUDA;
  const int64_t ld = default_ld(batch);
  const int c = host_chunk(T);
  for (int q0 = 0; q0 < T; q0 += c) {
    const int n = T - q0 < c ? T - q0 : c;
    const size_t o_qi = static_cast<size_t>(q0) * H_I * DSA_D_INDEX, o_w = static_cast<size_t>(q0) * H_I;
    const size_t o_q = static_cast<size_t>(q0) * H * DSA_D_QK, o_o = static_cast<size_t>(q0) * H * DSA_D_V;
    if (cudaMemcpyAsync(q_idx + o_qi, h_q_idx + o_qi, static_cast<size_t>(n) * H_I * DSA_D_INDEX,
                        cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
        cudaMemcpyAsync(w + o_w, h_w + o_w, static_cast<size_t>(n) * H_I * sizeof(float), cudaMemcpyHostToDevice,
                        s_in) != cudaSuccess ||
        cudaMemcpyAsync(q + o_q, h_q + o_q, static_cast<size_t>(n) * H * DSA_D_QK * 2, cudaMemcpyHostToDevice,
                        s_in) != cudaSuccess ||
        !order_after(E, s_in, s_cp))
      return DSA_ERR_CUDA;
    const dsa_batch sub = chunk_batch(batch, q0, n);
    const WsLayout L = layout(ws, DSA_OP_FORWARD, &sub, H, k, ld);
    dsa_status st = run_indexer(&sub, q_idx + o_qi, k_idx, w + o_w, H_I, L.scores, ld, L, s_cp);
    if (st == DSA_OK) st = run_topk(&sub, L.scores, ld, k, L.idx, L, s_cp);
    if (st == DSA_OK)
      st = run_mla(&sub, q + o_q, kv, L.idx, k, H, sm_scale, out + o_o, lse ? lse + static_cast<size_t>(q0) * H : nullptr,
                   L, s_cp);
    if (st != DSA_OK) return st;
    if (!order_after(E, s_cp, s_out) ||
        cudaMemcpyAsync(h_out + o_o, out + o_o, static_cast<size_t>(n) * H * DSA_D_V * 2, cudaMemcpyDeviceToHost,
                        s_out) != cudaSuccess)
      return DSA_ERR_CUDA;
  }
  return order_after(E, s_out, s_cp) ? DSA_OK : DSA_ERR_CUDA;
}

dsa_status dsa_forward_ws_views(const dsa_batch* batch, int H_I, int H, int k, void* ws, float** scores, int64_t* ld,
                                int32_t** idx) {
  (void)H_I;
  if (!batch_ok(batch) || !ws || !scores || !ld || !idx || !h_ok(H) || !k_ok(k)) return DSA_ERR_INVALID_ARGUMENT;
  const int64_t l = default_ld(batch);
  const WsLayout L = layout(ws, DSA_OP_FORWARD, batch, H, k, l);
  *scores = L.scores;
  *ld = l;
  *idx = L.idx;
  return DSA_OK;
}

dsa_status dsa_read_device_status(const void* ws, uint32_t* flags, void* stream) {
  if (!ws || !flags) return DSA_ERR_INVALID_ARGUMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess) return DSA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
  *flags = v;
  return v == 0 ? DSA_OK : DSA_ERR_DEVICE;
}

const char* dsa_status_string(dsa_status s) {
  switch (s) {
    case DSA_OK: return "DSA_OK";
    case DSA_ERR_INVALID_ARGUMENT: return "DSA_ERR_INVALID_ARGUMENT";
    case DSA_ERR_UNSUPPORTED: return "DSA_ERR_UNSUPPORTED";
    case DSA_ERR_WORKSPACE_TOO_SMALL: return "DSA_ERR_WORKSPACE_TOO_SMALL";
    case DSA_ERR_CUDA: return "DSA_ERR_CUDA";
    case DSA_ERR_DEVICE: return "DSA_ERR_DEVICE";
  }
  return "DSA_ERR_UNKNOWN";
}

int dsa_abi_version(void) { return DSA_ABI_VERSION; }

uint64_t dsa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"

// ----------------------------------------------------------------------------
// Indexer without a caller workspace: the plan and status word live in a
// fixed device array of this file (sized for DSA_NOALLOC_MAX_Q queries).
namespace {
// Header plus the indexer plan of DSA_NOALLOC_MAX_Q queries, padded exactly as
// plan_bytes() pads it, so that a call at the limit fits.
constexpr size_t kNoAllocBytes =
    kWsHeader + ((6 * static_cast<size_t>(DSA_NOALLOC_MAX_Q) + 2) * sizeof(int32_t) + kAlign - 1) / kAlign * kAlign;
}  // namespace

// In host code this name stands for the array, not for a device address; the
// kernels get the address that cudaGetSymbolAddress returns on each device.
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocBytes];

namespace {
void* noalloc_scratch_on_current_device() {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}
}  // namespace

extern "C" dsa_status dsa_indexer_scores_noalloc(const dsa_batch* batch, const uint8_t* q_idx,
                                                 const uint8_t* k_idx, const float* w, int H_I, float* scores,
                                                 int64_t ld, void* stream) {
  if (!batch_ok(batch)) return DSA_ERR_INVALID_ARGUMENT;
  if (batch->num_q > 0 && (!q_idx || !k_idx || !w || !scores)) return DSA_ERR_INVALID_ARGUMENT;
  if (!hi_ok(H_I) || !paging_ok(batch)) return DSA_ERR_UNSUPPORTED;
  if (batch->num_q > DSA_NOALLOC_MAX_Q) return DSA_ERR_UNSUPPORTED;
  if (ld < batch->max_kv_len || ld % 4 != 0) return DSA_ERR_UNSUPPORTED;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(w) || !aligned16(scores)) return DSA_ERR_UNSUPPORTED;
  void* ws = noalloc_scratch_on_current_device();
  if (!ws) return DSA_ERR_CUDA;
  const WsLayout L = layout(ws, DSA_OP_INDEXER, batch, 8, 1, ld);
  if (L.bytes > kNoAllocBytes) return DSA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(L.status, 0, sizeof(uint32_t), st) != cudaSuccess) return DSA_ERR_CUDA;   // starts at zero
  return run_indexer(batch, q_idx, k_idx, w, H_I, scores, ld, L, st);
}
