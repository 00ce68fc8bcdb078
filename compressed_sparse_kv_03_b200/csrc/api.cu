// C-ABI entry points: argument validation, workspace layout, dispatch.
//
// Nothing here computes any part of the method; every step runs in the
// kernels.  Validation happens before anything is enqueued, so an argument
// error leaves the stream untouched.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <string>

#include "kernels.h"

namespace csa {

namespace {

thread_local std::string g_last_error;
std::atomic<uint64_t> g_launches{0};
std::atomic<int32_t> g_attn_kernel{0};
std::atomic<int32_t> g_batch_invariant{0};
std::atomic<int32_t> g_timeout_test{0};
struct EventPair {
  cudaEvent_t begin = nullptr, end = nullptr;
};
EventPair g_events[kNumKernelIds];

csa_status_t fail(csa_status_t st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

csa_status_t cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return CSA_OK;
  return fail(CSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr int kNumSMs = 148;           // B200: workspace layouts are sized for it
constexpr int kAttnTargetCtas = 2 * kNumSMs;
constexpr int kD = 128;
constexpr int kMaxWindow = 1024;
constexpr size_t kIndexerChunkBytes = size_t(512) << 20;   // score scratch per chunk of queries

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Indexer workspace: header | per query tau, candidate count and fallback
// list entry [3][chunk] u32 + the fallback count | work counter | candidates
// [chunk, cap] (key, entry) pairs | sampled keys [chunk, kPSampleKeys] u32 (the
// tensor-core scorers' sample passes).  O(top_k) per query: no score matrix
// is stored.
// Queries are processed in chunks so that the scratch stays bounded.
struct IndexerLayout {
  bool many;
  int64_t chunk, cap;
  size_t meta_off, counter_off, data_off, sample_off, total;
};

// Candidate slots per query: the sample aims at about 2 top_k keys reaching
// the threshold; twice that (and at least 8192) leaves room for its spread.
int64_t candidate_cap(int32_t top_k) {
  int64_t cap = 4 * (int64_t)(top_k > 0 ? top_k : 1);
  if (cap < 8192) cap = 8192;
  return (cap + 255) / 256 * 256;
}

IndexerLayout indexer_layout(int64_t T, int64_t max_entries, int32_t top_k) {
  IndexerLayout l;
  l.many = T > kFusedMaxQueries && max_entries <= kManyMaxEntries;
  l.cap = candidate_cap(top_k);
  const int64_t per_query = l.cap * 8 + 12 + kPSampleKeys * 4;
  int64_t c = (int64_t)(kIndexerChunkBytes / per_query);
  if (c > 65535) c = 65535;
  if (!l.many && c > kFusedMaxQueries) c = kFusedMaxQueries;
  c &= ~int64_t(255);   // chunk starts stay aligned for the scorers' weight loads
  if (c < 256) c = 256;
  l.chunk = c < T ? c : T;
  if (l.chunk < 1) l.chunk = 1;
  l.meta_off = kWsHeader;
  l.counter_off = l.meta_off + align256(((size_t)l.chunk * 3 + 1) * sizeof(uint32_t));
  l.data_off = l.counter_off + 256;
  l.sample_off = l.data_off + align256((size_t)l.chunk * l.cap * 8);
  l.total = l.sample_off + align256((size_t)l.chunk * kPSampleKeys * 4);
  return l;
}

struct Split {
  int n, len;
};
// Split-KV layout for T queries whose row lists hold at most total_max rows.
Split attn_split(int64_t T, int64_t total_max, int H) {
  const int64_t hgroups = (H + 63) / 64;
  const int64_t ctas = T * hgroups;
  int64_t max_split = (total_max + 127) / 128;
  if (max_split < 1) max_split = 1;
  int64_t n = (kAttnTargetCtas + ctas - 1) / ctas;
  if (n > max_split) n = max_split;
  if (n < 1) n = 1;
  int64_t len = (total_max + n - 1) / n;
  len = (len + 127) / 128 * 128;
  if (len < 128) len = 128;
  n = (total_max + len - 1) / len;
  if (n < 1) n = 1;
  return Split{(int)n, (int)len};
}

// Split for the persistent tensor-core kernel: at most one work item per SM
// (a 64-head group of one query over one slice), slices of whole 128-row tiles
// as even as possible.  Never more slices than `ws` (the workspace layout).
Split attn_split_tc(int64_t T, int64_t total_max, int H, const Split& ws) {
  const int64_t q_items = T * ((H + 63) / 64);
  const int64_t tiles = (total_max + 127) / 128;
  int64_t n_max = q_items >= kNumSMs ? 1 : kNumSMs / q_items;
  if (n_max > ws.n) n_max = ws.n;
  if (n_max <= 1 || tiles <= 1) return Split{1, (int)(tiles * 128 > 128 ? tiles * 128 : 128)};
  const int64_t len_tiles = (tiles + n_max - 1) / n_max;
  const int64_t n = (tiles + len_tiles - 1) / len_tiles;
  return Split{(int)n, (int)(len_tiles * 128)};
}

// Split for the head-dim-512 kernel (CTAs of 32 heads, two resident per SM):
// slices of whole 64-row spans, as many as fit in one wave of CTAs and never
// more than `ws`.  Each slice costs a partial O of 2 KB per head written and
// merged, so the split stops at one wave (B = 64, H = 64, 1152 rows: 134 us
// at two slices against 150 us unsplit).
Split attn_split_512(int64_t T, int64_t total_max, int H, const Split& ws) {
  const int64_t ctas = T * ((H + 31) / 32);
  const int64_t tiles = (total_max + 63) / 64;
  int64_t n = 2 * kNumSMs / ctas;
  if (n > ws.n) n = ws.n;
  if (n > tiles) n = tiles;
  if (n <= 1 || tiles <= 1) return Split{1, (int)(tiles * 64 > 64 ? tiles * 64 : 64)};
  const int64_t len_tiles = (tiles + n - 1) / n;
  return Split{(int)((tiles + len_tiles - 1) / len_tiles), (int)(len_tiles * 64)};
}

// Batch-invariant decode: fixed 512-row slices of every query's row list.
constexpr int kInvariantSliceRows = 512;
Split attn_split_invariant(int64_t total_max) {
  int64_t n = (total_max + kInvariantSliceRows - 1) / kInvariantSliceRows;
  if (n < 1) n = 1;
  return Split{(int)n, kInvariantSliceRows};
}

size_t attn_partials_bytes(int64_t T, int H, int n, int d = kD) {
  if (n == 1) return kWsHeader;
  const size_t acc = (size_t)T * n * H * d * sizeof(float);
  const size_t ml = (size_t)T * n * H * 2 * sizeof(float);
  return kWsHeader + align256(acc) + align256(ml);
}

// Workspace of a decode call: the mma.sync split (which bounds the tcgen05
// one) and, in batch-invariant mode, the fixed slices.
size_t attn_ws_bytes(int64_t T, int H, int64_t total_max, int d = kD) {
  size_t b = attn_partials_bytes(T, H, attn_split(T, total_max, H).n, d);
  if (g_batch_invariant.load(std::memory_order_relaxed)) {
    const size_t bi = attn_partials_bytes(T, H, attn_split_invariant(total_max).n, d);
    if (bi > b) b = bi;
  }
  return b;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

csa_status_t check_cache(const csa_cache_t* c, const char* name) {
  if (c == nullptr || c->data == nullptr) return fail(CSA_ERR_INVALID_ARG, "%s: null cache", name);
  if (!aligned16(c->data)) return fail(CSA_ERR_INVALID_ARG, "%s: data not 16-byte aligned", name);
  if (c->n_rows <= 0) return fail(CSA_ERR_INVALID_ARG, "%s: n_rows must be > 0", name);
  if (c->page_table != nullptr) {
    if (c->page_size <= 0 || c->max_pages <= 0)
      return fail(CSA_ERR_INVALID_ARG, "%s: page_size and max_pages must be > 0", name);
  } else if (c->seq_stride < 0) {
    return fail(CSA_ERR_INVALID_ARG, "%s: seq_stride must be >= 0", name);
  }
  return CSA_OK;
}

CacheRef to_ref(const csa_cache_t* c) {
  CacheRef r;
  r.data = static_cast<const __nv_bfloat16*>(c->data);
  r.n_rows = c->n_rows;
  r.seq_stride = c->seq_stride;
  r.page_table = c->page_table;
  r.page_size = c->page_table ? c->page_size : 1;
  r.max_pages = c->page_table ? c->max_pages : 0;
  return r;
}

csa_status_t check_ws(void* ws, size_t ws_bytes, size_t need, const char* name) {
  if (need == 0) return CSA_OK;
  if (ws == nullptr || ws_bytes < need)
    return fail(CSA_ERR_WORKSPACE, "%s: workspace of %zu bytes needed, %zu given", name, need,
                ws_bytes);
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return fail(CSA_ERR_WORKSPACE, "%s: workspace must be 256-byte aligned", name);
  return CSA_OK;
}

}  // namespace

namespace {
// Inside stream capture an event becomes a graph node only when recorded as
// an external event; outside capture this is a plain record.
void record_event(cudaEvent_t ev, cudaStream_t stream) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(stream, &cs);
  if (cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(ev, stream, cudaEventRecordExternal);
  else
    cudaEventRecord(ev, stream);
}
}  // namespace

void set_last_error(const char* msg) { g_last_error = msg; }

int32_t attention_kernel_choice() { return g_attn_kernel.load(std::memory_order_relaxed); }

bool take_attention_timeout_test() { return g_timeout_test.exchange(0, std::memory_order_relaxed) != 0; }

void Launch::begin(int32_t kernel) const {
  const EventPair& e = g_events[kernel];
  if (e.begin) record_event(e.begin, stream);
}

cudaError_t Launch::end(int32_t kernel) const {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  cudaError_t err = cudaGetLastError();
  const EventPair& e = g_events[kernel];
  if (e.end) record_event(e.end, stream);
  return err;
}

}  // namespace csa

using namespace csa;

extern "C" {

const char* csa_version(void) { return "csa-b200 0.1 (sm_100a)"; }

const char* csa_last_error(void) { return g_last_error.c_str(); }

uint64_t csa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

csa_status_t csa_set_attention_kernel(int32_t choice) {
  if (choice < 0 || choice > 2)
    return fail(CSA_ERR_INVALID_ARG, "csa_set_attention_kernel: choice %d out of range", choice);
  g_attn_kernel.store(choice, std::memory_order_relaxed);
  return CSA_OK;
}

csa_status_t csa_test_attention_timeout(int32_t on) {
  if (on != 0 && on != 1)
    return fail(CSA_ERR_INVALID_ARG, "csa_test_attention_timeout: on must be 0 or 1, got %d", on);
  g_timeout_test.store(on, std::memory_order_relaxed);
  return CSA_OK;
}

csa_status_t csa_set_batch_invariant(int32_t on) {
  if (on != 0 && on != 1)
    return fail(CSA_ERR_INVALID_ARG, "csa_set_batch_invariant: on must be 0 or 1, got %d", on);
  g_batch_invariant.store(on, std::memory_order_relaxed);
  return CSA_OK;
}

csa_status_t csa_set_timing_events(int32_t kernel_id, void* ev_begin, void* ev_end) {
  if (kernel_id < 0 || kernel_id >= kNumKernelIds)
    return fail(CSA_ERR_INVALID_ARG, "csa_set_timing_events: kernel_id %d out of range", kernel_id);
  if ((ev_begin == nullptr) != (ev_end == nullptr))
    return fail(CSA_ERR_INVALID_ARG, "csa_set_timing_events: give both events or neither");
  g_events[kernel_id].begin = static_cast<cudaEvent_t>(ev_begin);
  g_events[kernel_id].end = static_cast<cudaEvent_t>(ev_end);
  return CSA_OK;
}

// ---- workspace -------------------------------------------------------------
size_t csa_indexer_topk_workspace_size(int64_t T, int64_t max_entries, int32_t top_k) {
  if (T <= 0 || max_entries < 0) return kWsHeader;
  return indexer_layout(T, max_entries, top_k).total;
}

size_t csa_sparse_attn_decode_workspace_size(int32_t B, int32_t H, int32_t d, int32_t top_k,
                                             int32_t window) {
  if (B <= 0 || H <= 0) return kWsHeader;
  return attn_ws_bytes(B, H, (int64_t)top_k + window, d == 512 ? 512 : kD);
}

size_t csa_sparse_attn_prefill_workspace_size(int64_t L, int32_t H, int32_t d) {
  (void)L; (void)H; (void)d;
  return kWsHeader;   // prefill never splits a query's row list
}

size_t hca_attn_workspace_size(int64_t T, int32_t H, int32_t d, int64_t max_entries,
                               int32_t window) {
  if (T <= 0 || H <= 0) return kWsHeader;
  return attn_ws_bytes(T, H, max_entries + window, d == 512 ? 512 : kD);
}

csa_status_t csa_workspace_init(void* ws, size_t ws_bytes, csa_stream_t stream) {
  if (ws == nullptr || ws_bytes < kWsHeader)
    return fail(CSA_ERR_WORKSPACE, "csa_workspace_init: workspace smaller than its header");
  return cuda_status(cudaMemsetAsync(ws, 0, kWsHeader, (cudaStream_t)stream), "cudaMemsetAsync");
}

csa_status_t csa_workspace_check(void* ws, csa_stream_t stream) {
  if (ws == nullptr) return fail(CSA_ERR_WORKSPACE, "csa_workspace_check: null workspace");
  WsHeader h;
  cudaError_t e = cudaMemcpyAsync(&h, ws, sizeof(h), cudaMemcpyDeviceToHost, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_status(e, "csa_workspace_check");
  if (h.code == kErrNone) return CSA_OK;
  static const char* names[] = {"none", "entry index outside the cache",
                                "page id outside the pool", "eligible entries above max_entries",
                                "window length outside [0, window]",
                                "a bounded pipeline wait timed out",
                                "top-k scratch inconsistent"};
  const char* what = (h.code > 0 && h.code <= 6) ? names[h.code] : "unknown";
  fail(CSA_ERR_DEVICE_CHECK, "device check: %s (query %d, value %lld)", what, h.where,
       (long long)h.value);
  e = cudaMemsetAsync(ws, 0, kWsHeader, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  return CSA_ERR_DEVICE_CHECK;
}

// ---- step 1 ------------------------------------------------------------------
csa_status_t csa_compress_kv(const csa_bf16* C_a, const csa_bf16* Z_a, const csa_bf16* C_b,
                             const csa_bf16* Z_b, const float* bias, int64_t n_tokens,
                             int32_t dim, int32_t m, int32_t overlap, csa_bf16* out,
                             csa_stream_t stream) {
  if (n_tokens < 0 || m < 1 || dim < 8 || dim % 8 != 0 || (overlap != 0 && overlap != 1))
    return fail(CSA_ERR_INVALID_ARG,
                "csa_compress_kv: need n_tokens >= 0, m >= 1, dim a positive multiple of 8, "
                "overlap in {0,1} (got %lld, %d, %d, %d)",
                (long long)n_tokens, m, dim, overlap);
  if (n_tokens / m == 0) return CSA_OK;   // no complete block: nothing to write
  if (C_a == nullptr || Z_a == nullptr || out == nullptr)
    return fail(CSA_ERR_INVALID_ARG, "csa_compress_kv: C_a, Z_a and out are required");
  if (!aligned16(C_a) || !aligned16(Z_a) || !aligned16(out) || (C_b && !aligned16(C_b)) ||
      (Z_b && !aligned16(Z_b)) || (bias && !aligned16(bias)))
    return fail(CSA_ERR_INVALID_ARG, "csa_compress_kv: tensors must be 16-byte aligned");
  Launch L{(cudaStream_t)stream};
  return cuda_status(
      launch_compress(L, (const __nv_bfloat16*)C_a, (const __nv_bfloat16*)Z_a,
                      (const __nv_bfloat16*)C_b, (const __nv_bfloat16*)Z_b, bias, n_tokens, dim, m,
                      overlap, (__nv_bfloat16*)out),
      "csa_compress_kv launch");
}

csa_status_t csa_cache_append(const csa_bf16* C_a, const csa_bf16* Z_a, const csa_bf16* C_b,
                              const csa_bf16* Z_b, const float* bias, const int64_t* pos,
                              int32_t B, int32_t dim, int32_t m, int32_t overlap,
                              csa_bf16* blk_c, csa_bf16* blk_z, csa_bf16* bb_c, csa_bf16* bb_z,
                              csa_bf16* win, int32_t window, const csa_cache_t* cache,
                              int64_t max_entries, void* ws, size_t ws_bytes, csa_stream_t stream) {
  const char* name = "csa_cache_append";
  if (B < 0 || m < 1 || dim < 8 || dim % 8 != 0 || dim > 2048 || window < 0 || max_entries < 0 ||
      (overlap != 0 && overlap != 1))
    return fail(CSA_ERR_INVALID_ARG,
                "%s: need B >= 0, m >= 1, dim a multiple of 8 in [8, 2048], window >= 0, "
                "max_entries >= 0, overlap in {0,1}", name);
  if (B == 0) return CSA_OK;
  if (C_a == nullptr || Z_a == nullptr || pos == nullptr || blk_c == nullptr || blk_z == nullptr)
    return fail(CSA_ERR_INVALID_ARG, "%s: C_a, Z_a, pos, blk_c and blk_z are required", name);
  if (overlap && (bb_c == nullptr || bb_z == nullptr))
    return fail(CSA_ERR_INVALID_ARG, "%s: overlap mode needs bb_c and bb_z", name);
  if (window > 0 && win == nullptr) return fail(CSA_ERR_INVALID_ARG, "%s: window > 0 needs win", name);
  csa_status_t st = check_cache(cache, name);
  if (st != CSA_OK) return st;
  if (!aligned16(C_a) || !aligned16(Z_a) || (C_b && !aligned16(C_b)) || (Z_b && !aligned16(Z_b)) ||
      (bias && !aligned16(bias)) || !aligned16(blk_c) || !aligned16(blk_z) ||
      (bb_c && !aligned16(bb_c)) || (bb_z && !aligned16(bb_z)) || (win && !aligned16(win)))
    return fail(CSA_ERR_INVALID_ARG, "%s: tensors must be 16-byte aligned", name);
  if ((st = check_ws(ws, ws_bytes, kWsHeader, name)) != CSA_OK) return st;
  CacheAppendArgs a{};
  a.Ca = (const __nv_bfloat16*)C_a;
  a.Za = (const __nv_bfloat16*)Z_a;
  a.Cb = (const __nv_bfloat16*)C_b;
  a.Zb = (const __nv_bfloat16*)Z_b;
  a.bias = bias;
  a.pos = pos;
  a.B = B;
  a.dim = dim;
  a.m = m;
  a.overlap = overlap;
  a.blk_c = (__nv_bfloat16*)blk_c;
  a.blk_z = (__nv_bfloat16*)blk_z;
  a.bb_c = (__nv_bfloat16*)bb_c;
  a.bb_z = (__nv_bfloat16*)bb_z;
  a.win = (__nv_bfloat16*)win;
  a.window = window;
  a.cache = to_ref(cache);
  a.max_entries = max_entries;
  a.err = static_cast<WsHeader*>(ws);
  Launch L{(cudaStream_t)stream};
  return cuda_status(launch_cache_append(L, a), "csa_cache_append launch");
}

csa_status_t csa_norm_rope(const csa_bf16* x, csa_bf16* out, int64_t T, int32_t H, int32_t dim,
                           const float* gain, float eps, const int64_t* pos, int64_t pos_mul,
                           int32_t rope_dims, float rope_base, int32_t inverse,
                           csa_stream_t stream) {
  const char* name = "csa_norm_rope";
  if (T < 0 || H < 1 || (dim != 64 && dim != 128 && dim != 256) || rope_dims < 0 ||
      rope_dims > dim || rope_dims % 8 != 0 || (inverse != 0 && inverse != 1) ||
      (rope_dims > 0 && !(rope_base > 1.f)) || !(eps == eps))
    return fail(CSA_ERR_INVALID_ARG,
                "%s: need T >= 0, H >= 1, dim in {64,128,256}, rope_dims a multiple of 8 <= dim, "
                "rope_base > 1, inverse in {0,1}", name);
  if (T == 0) return CSA_OK;
  if (x == nullptr || out == nullptr) return fail(CSA_ERR_INVALID_ARG, "%s: x and out are required", name);
  if (!aligned16(x) || !aligned16(out) || (gain && !aligned16(gain)))
    return fail(CSA_ERR_INVALID_ARG, "%s: tensors must be 16-byte aligned", name);
  NormRopeArgs a{};
  a.x = (const __nv_bfloat16*)x;
  a.out = (__nv_bfloat16*)out;
  a.T = T;
  a.H = H;
  a.dim = dim;
  a.gain = gain;
  a.eps = eps;
  a.pos = pos;
  a.pos_mul = pos_mul;
  a.rope_dims = rope_dims;
  a.rope_base = rope_base;
  a.inverse = inverse;
  Launch L{(cudaStream_t)stream};
  return cuda_status(launch_norm_rope(L, a), "csa_norm_rope launch");
}

// ---- steps 2-3 ---------------------------------------------------------------
namespace {

// Score + select, one chunk of queries at a time: a threshold from a sample
// of each query's scores, scoring into candidate lists, exact finish.  Few
// queries (decode): a per-query sample launch and one CTA per query in the
// finish.  Many queries (prefill): the tcgen05 scorer's own sample pass, a
// per-warp threshold and finish, when its shapes allow.  `base` carries the
// query / key operands.
csa_status_t run_indexer_topk(IndexerArgs base, const int64_t* q_pos, int64_t T, int32_t m,
                              int64_t max_entries, int32_t top_k, int32_t* idx_out,
                              int32_t* count_out, float* score_out, void* ws, csa_stream_t stream) {
  Launch L{(cudaStream_t)stream};
  const IndexerLayout lay = indexer_layout(T, max_entries, top_k);
  char* wsb = static_cast<char*>(ws);
  WsHeader* hdr = static_cast<WsHeader*>(ws);
  uint32_t* work = reinterpret_cast<uint32_t*>(wsb + lay.counter_off);
  for (int64_t t0 = 0; t0 < T; t0 += lay.chunk) {
    const int64_t n = T - t0 < lay.chunk ? T - t0 : lay.chunk;
    IndexerArgs ia = base;
    ia.q_pos = q_pos;
    ia.T = T;
    ia.m = m;
    ia.max_entries = max_entries;
    ia.t_begin = t0;
    ia.work = work;
    ia.err = hdr;
    cudaError_t e;
    uint32_t* meta = reinterpret_cast<uint32_t*>(wsb + lay.meta_off);
    ia.tau = meta;
    ia.cand_count = meta + lay.chunk;
    ia.fb_list = meta + 2 * lay.chunk;
    ia.fb_count = meta + 3 * lay.chunk;
    ia.cand = reinterpret_cast<uint2*>(wsb + lay.data_off);
    ia.cand_cap = lay.cap;
    ia.skip_le = score_out ? 0 : top_k;   // scores of all-selected queries still come from the scorer
    ia.psample = reinterpret_cast<uint32_t*>(wsb + lay.sample_off);
    if (lay.many && tc_indexer_prefill_supported(ia, n) && topk_many_supported(ia)) {
      // the scorer's sample pass, thresholds (which zero the counts and the
      // work counter), the scorer's candidate pass, per-warp finish
      // (no sample pass when every query's entries fit its candidate list:
      // the thresholds are then all zero)
      e = cudaMemsetAsync(work, 0, sizeof(uint32_t), L.stream);
      if (e != cudaSuccess) return cuda_status(e, "indexer work counter memset");
      if (2 * max_entries > ia.cand_cap && (e = launch_indexer_scores_tc_prefill(L, ia, n, true)) != cudaSuccess)
        return cuda_status(e, "indexer sample launch");
      if ((e = launch_topk_threshold_many(L, ia, top_k, n, 128 / ia.H_I)) != cudaSuccess)
        return cuda_status(e, "top-k threshold launch");
      if ((e = launch_indexer_scores(L, ia, n)) != cudaSuccess) return cuda_status(e, "indexer score launch");
      if ((e = launch_topk_finish_many(L, ia, top_k, idx_out, count_out, score_out, n)) != cudaSuccess)
        return cuda_status(e, "top-k finish launch");
    } else if (tc_fp4_indexer_supported(ia, n)) {
      // 4-bit keys on the block-scaled tensor cores: the queries' operand
      // images (in the tail of the candidate area, whose per-query stride
      // shrinks by kFp4ImgSlots; this launch also zeroes the work counter),
      // the scorer's sample pass (whole chunks per query), one-warp
      // thresholds, its candidate pass
      ia.cand_cap = lay.cap - kFp4ImgSlots;
      ia.q_img = reinterpret_cast<uint8_t*>(wsb + lay.data_off) + (size_t)lay.chunk * (size_t)ia.cand_cap * 8;
      if ((e = launch_fp4_query_images(L, ia, n)) != cudaSuccess) return cuda_status(e, "query image launch");
      if ((e = launch_indexer_scores_fp4_tc(L, ia, n, true)) != cudaSuccess)
        return cuda_status(e, "indexer sample launch");
      if ((e = launch_topk_threshold_many(L, ia, top_k, n, 1)) != cudaSuccess)
        return cuda_status(e, "top-k threshold launch");
      if ((e = launch_indexer_scores_fp4_tc(L, ia, n, false)) != cudaSuccess)
        return cuda_status(e, "indexer score launch");
      if ((e = launch_topk_finish(L, ia, top_k, idx_out, count_out, score_out, n)) != cudaSuccess)
        return cuda_status(e, "top-k finish launch");
    } else {
      ia.psample = nullptr;
      // the work counter is zeroed before the sample launch (the scorer may
      // start while that one runs); the sample launch zeroes the counts
      e = cudaMemsetAsync(work, 0, sizeof(uint32_t), L.stream);
      if (e != cudaSuccess) return cuda_status(e, "indexer work counter memset");
      if ((e = launch_topk_sample(L, ia, top_k, n)) != cudaSuccess) return cuda_status(e, "top-k sample launch");
      if ((e = launch_indexer_scores(L, ia, n)) != cudaSuccess) return cuda_status(e, "indexer score launch");
      if ((e = launch_topk_finish(L, ia, top_k, idx_out, count_out, score_out, n)) != cudaSuccess)
        return cuda_status(e, "top-k finish launch");
    }
  }
  return CSA_OK;
}

// Checks shared by the bf16 and 4-bit indexer calls.
csa_status_t check_indexer_args(const char* name, int64_t T, int32_t H_I, int32_t c_I, int32_t m,
                                int64_t max_entries, int32_t top_k, const float* w,
                                const int32_t* idx_out, const int32_t* count_out,
                                const csa_cache_t* k_idx) {
  if (T < 0 || H_I < 1 || m < 1 || top_k < 1 || max_entries < 0)
    return fail(CSA_ERR_INVALID_ARG,
                "%s: need T >= 0, H_I >= 1, m >= 1, top_k >= 1, max_entries >= 0", name);
  if (T == 0) return CSA_OK;
  if (w == nullptr || idx_out == nullptr || count_out == nullptr)
    return fail(CSA_ERR_INVALID_ARG, "%s: w, idx_out and count_out are required", name);
  if (H_I > 64) return fail(CSA_ERR_UNSUPPORTED, "%s: H_I > 64 not built", name);
  if (c_I != 64 && c_I != 128)
    return fail(CSA_ERR_UNSUPPORTED, "%s: c_I must be 64 or 128 (got %d)", name, c_I);
  if (max_entries > kMaxSelectEntries)
    return fail(CSA_ERR_UNSUPPORTED, "%s: max_entries > %lld not built", name,
                (long long)kMaxSelectEntries);
  if (top_k > 4096) return fail(CSA_ERR_UNSUPPORTED, "%s: top_k > 4096 not built", name);
  return check_cache(k_idx, name);
}

}  // namespace

csa_status_t csa_indexer_topk(const csa_bf16* q_idx, const float* w, const csa_cache_t* k_idx,
                              const int32_t* seq_id, const int64_t* q_pos, int64_t T,
                              int32_t H_I, int32_t c_I, int32_t m, int64_t max_entries,
                              int32_t top_k, int32_t* idx_out, int32_t* count_out,
                              float* score_out, void* ws, size_t ws_bytes, csa_stream_t stream) {
  const char* name = "csa_indexer_topk";
  csa_status_t st =
      check_indexer_args(name, T, H_I, c_I, m, max_entries, top_k, w, idx_out, count_out, k_idx);
  if (st != CSA_OK || T == 0) return st;
  if (q_idx == nullptr) return fail(CSA_ERR_INVALID_ARG, "%s: q_idx is required", name);
  if (!aligned16(q_idx)) return fail(CSA_ERR_INVALID_ARG, "%s: q_idx alignment", name);
  const size_t need = csa_indexer_topk_workspace_size(T, max_entries, top_k);
  if ((st = check_ws(ws, ws_bytes, need, name)) != CSA_OK) return st;
  IndexerArgs ia;
  ia.q_idx = (const __nv_bfloat16*)q_idx;
  ia.w = w;
  ia.keys = to_ref(k_idx);
  ia.seq_id = seq_id;
  ia.H_I = H_I;
  ia.c_I = c_I;
  return run_indexer_topk(ia, q_pos, T, m, max_entries, top_k, idx_out, count_out, score_out, ws,
                          stream);
}

csa_status_t csa_quantize_mxfp4(const csa_bf16* x, int64_t n_vectors, int32_t dim, uint8_t* codes,
                                uint8_t* scales, csa_stream_t stream) {
  const char* name = "csa_quantize_mxfp4";
  if (n_vectors < 0 || dim < 32 || dim % 32 != 0)
    return fail(CSA_ERR_INVALID_ARG, "%s: need n_vectors >= 0 and dim a positive multiple of 32",
                name);
  if (n_vectors == 0) return CSA_OK;
  if (x == nullptr || codes == nullptr || scales == nullptr)
    return fail(CSA_ERR_INVALID_ARG, "%s: x, codes and scales are required", name);
  if (!aligned16(x) || !aligned16(codes))
    return fail(CSA_ERR_INVALID_ARG, "%s: x and codes must be 16-byte aligned", name);
  Launch L{(cudaStream_t)stream};
  return cuda_status(launch_mxfp4_quantize(L, (const __nv_bfloat16*)x, n_vectors * (dim / 32),
                                           codes, scales),
                     "csa_quantize_mxfp4 launch");
}

csa_status_t csa_indexer_topk_mxfp4(const csa_bf16* q_idx, const float* w,
                                    const csa_cache_t* k_codes, const uint8_t* k_scales,
                                    const int32_t* seq_id, const int64_t* q_pos, int64_t T,
                                    int32_t H_I, int32_t c_I, int32_t m, int64_t max_entries,
                                    int32_t top_k, int32_t* idx_out, int32_t* count_out,
                                    float* score_out, void* ws, size_t ws_bytes,
                                    csa_stream_t stream) {
  const char* name = "csa_indexer_topk_mxfp4";
  csa_status_t st =
      check_indexer_args(name, T, H_I, c_I, m, max_entries, top_k, w, idx_out, count_out, k_codes);
  if (st != CSA_OK || T == 0) return st;
  if (q_idx == nullptr || k_scales == nullptr)
    return fail(CSA_ERR_INVALID_ARG, "%s: q_idx and k_scales are required", name);
  if (!aligned16(q_idx) || !aligned16(k_scales))
    return fail(CSA_ERR_INVALID_ARG, "%s: q_idx and k_scales must be 16-byte aligned", name);
  const size_t need = csa_indexer_topk_workspace_size(T, max_entries, top_k);
  if ((st = check_ws(ws, ws_bytes, need, name)) != CSA_OK) return st;
  IndexerArgs ia;
  ia.q_idx = (const __nv_bfloat16*)q_idx;
  ia.w = w;
  ia.keys = to_ref(k_codes);
  ia.seq_id = seq_id;
  ia.H_I = H_I;
  ia.c_I = c_I;
  ia.fp4 = 1;
  ia.k_scales = k_scales;
  return run_indexer_topk(ia, q_pos, T, m, max_entries, top_k, idx_out, count_out, score_out, ws,
                          stream);
}

// ---- step 4 ------------------------------------------------------------------
namespace {

csa_status_t check_attn_common(const char* name, const csa_bf16* q, const csa_bf16* out,
                               int32_t H, int32_t d, int32_t window) {
  if (q == nullptr || out == nullptr) return fail(CSA_ERR_INVALID_ARG, "%s: q and out required", name);
  if (H < 1 || window < 0) return fail(CSA_ERR_INVALID_ARG, "%s: need H >= 1, window >= 0", name);
  if (d != kD && d != 512)
    return fail(CSA_ERR_UNSUPPORTED, "%s: head dim %d not built (128 or 512)", name, d);
  if (H > 128) return fail(CSA_ERR_UNSUPPORTED, "%s: H > 128 not built", name);
  if (window > kMaxWindow) return fail(CSA_ERR_UNSUPPORTED, "%s: window > %d", name, kMaxWindow);
  if (!aligned16(q) || !aligned16(out)) return fail(CSA_ERR_INVALID_ARG, "%s: q/out alignment", name);
  return CSA_OK;
}

// The fused query prologue / output epilogue: checks and AttnArgs fields.
csa_status_t apply_qrope(const char* name, const csa_qrope_t* r, bool decode, AttnArgs& a) {
  if (r == nullptr) return CSA_OK;
  if (r->rope_dims < 0 || r->rope_dims > kD || r->rope_dims % 8 != 0 ||
      (r->rope_dims > 0 && !(r->rope_base > 1.f)) || (r->derotate != 0 && r->derotate != 1) ||
      !(r->q_eps == r->q_eps))
    return fail(CSA_ERR_INVALID_ARG,
                "%s: qrope needs rope_dims a multiple of 8 up to %d, rope_base > 1 when rotating, "
                "derotate in {0,1}", name, kD);
  if (decode && r->rope_dims > 0 && r->pos == nullptr)
    return fail(CSA_ERR_INVALID_ARG, "%s: qrope on a decode call needs pos", name);
  if (r->q_gain != nullptr && !aligned16(r->q_gain))
    return fail(CSA_ERR_INVALID_ARG, "%s: qrope gain must be 16-byte aligned", name);
  a.qprologue = (r->q_eps >= 0.f || r->rope_dims > 0) ? 1 : 0;
  a.q_norm_gain = r->q_gain;
  a.q_norm_eps = r->q_eps;
  a.q_rope_dims = r->rope_dims;
  a.q_rope_base = r->rope_base;
  a.out_derotate = r->rope_dims > 0 ? r->derotate : 0;
  a.rope_pos = r->pos;
  return CSA_OK;
}

csa_status_t need_tc_for_qrope(const char* name, const AttnArgs& a) {
  if ((a.qprologue || a.out_derotate) && !a.use_tc)
    return fail(CSA_ERR_UNSUPPORTED,
                "%s: the fused query prologue / output de-rotation runs on the tensor-core "
                "attention kernel only", name);
  return CSA_OK;
}

}  // namespace

csa_status_t csa_sparse_attn_prefill(const csa_bf16* q, const csa_bf16* kv_comp,
                                     int64_t n_entries, const csa_bf16* kv_raw,
                                     const int32_t* idx, const int32_t* count, int64_t L,
                                     int32_t H, int32_t d, int32_t top_k, int32_t window,
                                     float sm_scale, const float* sink, csa_bf16* out,
                                     float* lse, void* ws, size_t ws_bytes,
                                     csa_stream_t stream, const csa_qrope_t* qrope) {
  const char* name = "csa_sparse_attn_prefill";
  if (L == 0) return CSA_OK;
  csa_status_t st = check_attn_common(name, q, out, H, d, window);
  if (st != CSA_OK) return st;
  if (kv_raw == nullptr || idx == nullptr || count == nullptr || L < 0 || top_k < 1 ||
      n_entries < 0 || (n_entries > 0 && kv_comp == nullptr))
    return fail(CSA_ERR_INVALID_ARG, "%s: kv_raw, idx, count required; L >= 0, top_k >= 1", name);
  if (L > 0x7fffffff) return fail(CSA_ERR_UNSUPPORTED, "%s: L >= 2^31", name);
  if (L == 0) return check_ws(ws, ws_bytes, kWsHeader, name);
  AttnArgs a{};
  a.d = d;
  a.q = (const __nv_bfloat16*)q;
  a.T = L;
  a.H = H;
  a.kv.data = (const __nv_bfloat16*)(kv_comp ? kv_comp : kv_raw);
  a.kv.n_rows = n_entries;
  a.kv.seq_stride = 0;
  a.kv.page_table = nullptr;
  a.kv.page_size = 1;
  a.kv.max_pages = 0;
  a.seq_per_query = 0;
  a.idx = idx;
  a.top_k = top_k;
  a.count = count;
  a.q_pos = nullptr;
  a.m = 1;
  a.max_entries = top_k;
  a.win = (const __nv_bfloat16*)kv_raw;
  a.win_len = nullptr;
  a.window = window;
  a.win_rows = L;
  a.sm_scale = sm_scale;
  a.sink = sink;
  a.out = (__nv_bfloat16*)out;
  a.lse = lse;
  if ((st = apply_qrope(name, qrope, false, a)) != CSA_OK) return st;
  // prefill: one slice per query (many queries fill the GPU)
  a.use_tc = attention_uses_tc(a);
  if ((st = need_tc_for_qrope(name, a)) != CSA_OK) return st;
  a.n_split = 1;
  a.split_len = (int)(((int64_t)top_k + window + 63) / 64 * 64);
  st = check_ws(ws, ws_bytes, kWsHeader, name);
  if (st != CSA_OK) return st;
  a.err = static_cast<WsHeader*>(ws);
  a.part_acc = a.part_ml = nullptr;
  Launch Lc{(cudaStream_t)stream};
  return cuda_status(launch_attention(Lc, a), name);
}

namespace {

// Split selection, workspace check and launch shared by the decode calls; `a`
// holds every field but the split / workspace ones.
csa_status_t run_decode_attention(AttnArgs a, const char* name, int32_t B, int32_t H,
                                  int32_t top_k, int32_t window, void* ws, size_t ws_bytes,
                                  csa_stream_t stream) {
  const Split sp_ws = attn_split(B, (int64_t)top_k + window, H);
  const bool invariant = g_batch_invariant.load(std::memory_order_relaxed) != 0;
  const Split sp_inv = attn_split_invariant((int64_t)top_k + window);
  const int n_need = invariant && sp_inv.n > sp_ws.n ? sp_inv.n : sp_ws.n;
  csa_status_t st = check_ws(ws, ws_bytes, attn_partials_bytes(B, H, n_need, a.d), name);
  if (st != CSA_OK) return st;
  a.use_tc = attention_uses_tc(a);
  if ((st = need_tc_for_qrope(name, a)) != CSA_OK) return st;
  const Split sp = invariant ? sp_inv
                   : a.use_tc ? attn_split_tc(B, (int64_t)top_k + window, H, sp_ws)
                   : a.d == 512 ? attn_split_512(B, (int64_t)top_k + window, H, sp_ws) : sp_ws;
  a.n_split = sp.n;
  a.split_len = sp.len;
  a.err = static_cast<WsHeader*>(ws);
  if (sp.n > 1) {
    char* p = static_cast<char*>(ws) + kWsHeader;
    a.part_acc = reinterpret_cast<float*>(p);
    a.part_ml = reinterpret_cast<float*>(p + align256((size_t)B * sp.n * H * a.d * sizeof(float)));
  }
  Launch L{(cudaStream_t)stream};
  return cuda_status(launch_attention(L, a), name);
}

AttnArgs decode_args(const csa_bf16* q, const csa_cache_t* kv, const csa_bf16* win,
                     const int32_t* win_len, const int32_t* idx, const int32_t* count, int32_t B,
                     int32_t H, int32_t top_k, int32_t window, float sm_scale, const float* sink,
                     csa_bf16* out, float* lse) {
  AttnArgs a{};
  a.q = (const __nv_bfloat16*)q;
  a.T = B;
  a.H = H;
  a.kv = to_ref(kv);
  a.seq_per_query = 1;
  a.idx = idx;
  a.top_k = top_k;
  a.count = count;
  a.q_pos = nullptr;
  a.m = 1;
  a.max_entries = top_k;
  a.win = (const __nv_bfloat16*)win;
  a.win_len = win_len;
  a.window = window;
  a.sm_scale = sm_scale;
  a.sink = sink;
  a.out = (__nv_bfloat16*)out;
  a.lse = lse;
  return a;
}

csa_status_t check_decode_args(const char* name, const csa_bf16* q, const csa_cache_t* kv,
                               const csa_bf16* win, const int32_t* win_len, const int32_t* idx,
                               const int32_t* count, int32_t B, int32_t H, int32_t d,
                               int32_t top_k, int32_t window, const csa_bf16* out) {
  csa_status_t st = check_attn_common(name, q, out, H, d, window);
  if (st != CSA_OK) return st;
  if ((st = check_cache(kv, name)) != CSA_OK) return st;
  if (idx == nullptr || count == nullptr || B < 0 || top_k < 1)
    return fail(CSA_ERR_INVALID_ARG, "%s: idx, count required; B >= 0, top_k >= 1", name);
  if (window > 0 && (win == nullptr || win_len == nullptr))
    return fail(CSA_ERR_INVALID_ARG, "%s: window > 0 needs win and win_len", name);
  return CSA_OK;
}

}  // namespace

}  // extern "C"

// Host-side argument checks of a decode attention call, for the entry points
// that wrap csa_sparse_attn_decode (internal linkage to the C ABI: not exported
// under a C name).
csa_status_t csa::check_decode_call(const char* name, const csa_bf16* q, const csa_cache_t* kv,
                                    const csa_bf16* win, const int32_t* win_len,
                                    const int32_t* idx, const int32_t* count, int32_t B,
                                    int32_t H, int32_t d, int32_t top_k, int32_t window,
                                    const csa_bf16* out) {
  return check_decode_args(name, q, kv, win, win_len, idx, count, B, H, d, top_k, window, out);
}

extern "C" {

csa_status_t csa_sparse_attn_decode(const csa_bf16* q, const csa_cache_t* kv_comp,
                                    const csa_bf16* win, const int32_t* win_len,
                                    const int32_t* idx, const int32_t* count, int32_t B,
                                    int32_t H, int32_t d, int32_t top_k, int32_t window,
                                    float sm_scale, const float* sink, csa_bf16* out,
                                    float* lse, void* ws, size_t ws_bytes,
                                    csa_stream_t stream, const csa_qrope_t* qrope) {
  const char* name = "csa_sparse_attn_decode";
  if (B == 0) return CSA_OK;
  csa_status_t st =
      check_decode_args(name, q, kv_comp, win, win_len, idx, count, B, H, d, top_k, window, out);
  if (st != CSA_OK) return st;
  AttnArgs a = decode_args(q, kv_comp, win, win_len, idx, count, B, H, top_k, window,
                           sm_scale, sink, out, lse);
  a.d = d;
  if ((st = apply_qrope(name, qrope, true, a)) != CSA_OK) return st;
  return run_decode_attention(a, name, B, H, top_k, window, ws, ws_bytes, stream);
}

csa_status_t csa_quantize_entries_fp8(const csa_bf16* x, int64_t n, int32_t dim, int32_t rope_dims,
                                      uint8_t* codes, uint8_t* scales, csa_bf16* rope,
                                      csa_stream_t stream) {
  const char* name = "csa_quantize_entries_fp8";
  if (n < 0 || dim < 8 || dim % 8 != 0 || rope_dims < 0 || rope_dims % 8 != 0 ||
      rope_dims >= dim || (dim - rope_dims) % 32 != 0)
    return fail(CSA_ERR_INVALID_ARG,
                "%s: need n >= 0, dim a multiple of 8, rope_dims a multiple of 8 below dim and "
                "dim - rope_dims a multiple of 32", name);
  if (n == 0) return CSA_OK;
  if (x == nullptr || codes == nullptr || scales == nullptr || (rope_dims > 0 && rope == nullptr))
    return fail(CSA_ERR_INVALID_ARG, "%s: x, codes, scales (and rope when rope_dims > 0) required",
                name);
  if (!aligned16(x) || !aligned16(codes) || (rope && !aligned16(rope)))
    return fail(CSA_ERR_INVALID_ARG, "%s: x, codes and rope must be 16-byte aligned", name);
  Launch L{(cudaStream_t)stream};
  return cuda_status(launch_fp8_entry_quantize(L, (const __nv_bfloat16*)x, n, dim, rope_dims,
                                               codes, scales, (__nv_bfloat16*)rope),
                     name);
}

csa_status_t csa_sparse_attn_decode_fp8(const csa_bf16* q, const csa_cache_t* kv_codes,
                                        const uint8_t* kv_scales, const csa_bf16* kv_rope,
                                        int32_t rope_dims, const csa_bf16* win,
                                        const int32_t* win_len, const int32_t* idx,
                                        const int32_t* count, int32_t B, int32_t H, int32_t d,
                                        int32_t top_k, int32_t window, float sm_scale,
                                        const float* sink, csa_bf16* out, float* lse, void* ws,
                                        size_t ws_bytes, csa_stream_t stream) {
  const char* name = "csa_sparse_attn_decode_fp8";
  if (B == 0) return CSA_OK;
  csa_status_t st =
      check_decode_args(name, q, kv_codes, win, win_len, idx, count, B, H, d, top_k, window, out);
  if (st != CSA_OK) return st;
  if (d != kD) return fail(CSA_ERR_UNSUPPORTED, "%s: mixed-precision entries at head dim 128 only", name);
  if (rope_dims < 0 || rope_dims % 8 != 0 || rope_dims >= kD || (kD - rope_dims) % 32 != 0)
    return fail(CSA_ERR_INVALID_ARG,
                "%s: rope_dims must be a multiple of 8 below 128 with 128 - rope_dims a multiple "
                "of 32 (got %d)", name, rope_dims);
  if (kv_scales == nullptr || (rope_dims > 0 && kv_rope == nullptr))
    return fail(CSA_ERR_INVALID_ARG, "%s: kv_scales (and kv_rope when rope_dims > 0) required", name);
  if (kv_rope && !aligned16(kv_rope))
    return fail(CSA_ERR_INVALID_ARG, "%s: kv_rope must be 16-byte aligned", name);
  AttnArgs a = decode_args(q, kv_codes, win, win_len, idx, count, B, H, top_k, window, sm_scale,
                           sink, out, lse);
  a.kv_fp8 = 1;
  a.kv_scales = kv_scales;
  a.kv_rope = (const __nv_bfloat16*)kv_rope;
  a.rope_dims = rope_dims;
  return run_decode_attention(a, name, B, H, top_k, window, ws, ws_bytes, stream);
}

csa_status_t hca_attn(const csa_bf16* q, const csa_cache_t* kv_comp, const csa_bf16* kv_win,
                      const int32_t* win_len, const int32_t* seq_id, const int64_t* q_pos,
                      int64_t T, int32_t H,
                      int32_t d, int32_t m, int64_t max_entries, int32_t window,
                      float sm_scale, const float* sink, csa_bf16* out, float* lse, void* ws,
                      size_t ws_bytes, csa_stream_t stream, const csa_qrope_t* qrope) {
  const char* name = "hca_attn";
  if (T == 0) return CSA_OK;
  csa_status_t st = check_attn_common(name, q, out, H, d, window);
  if (st != CSA_OK) return st;
  if ((st = check_cache(kv_comp, name)) != CSA_OK) return st;
  if (T < 0 || m < 1 || max_entries < 0)
    return fail(CSA_ERR_INVALID_ARG, "%s: need T >= 0, m >= 1, max_entries >= 0", name);
  if (win_len != nullptr && q_pos == nullptr)
    return fail(CSA_ERR_INVALID_ARG, "%s: decode (win_len given) needs q_pos", name);
  if (window > 0 && kv_win == nullptr)
    return fail(CSA_ERR_INVALID_ARG, "%s: window > 0 needs kv_win", name);
  if (T > 0x7fffffff) return fail(CSA_ERR_UNSUPPORTED, "%s: T >= 2^31", name);
  if (T == 0) return check_ws(ws, ws_bytes, kWsHeader, name);
  AttnArgs a{};
  a.d = d;
  a.q = (const __nv_bfloat16*)q;
  a.T = T;
  a.H = H;
  a.kv = to_ref(kv_comp);
  a.seq_per_query = win_len != nullptr ? 1 : 0;
  a.seq_id = seq_id;
  a.idx = nullptr;
  a.top_k = 0;
  a.count = nullptr;
  a.q_pos = q_pos;
  a.m = m;
  a.max_entries = max_entries;
  a.win = (const __nv_bfloat16*)kv_win;
  a.win_len = win_len;
  a.window = window;
  // raw rows known: all T of them when query i is row i (no q_pos, or packed)
  a.win_rows = (win_len == nullptr && (q_pos == nullptr || seq_id != nullptr)) ? T : 0;
  a.sm_scale = sm_scale;
  a.sink = sink;
  a.out = (__nv_bfloat16*)out;
  a.lse = lse;
  if ((st = apply_qrope(name, qrope, false, a)) != CSA_OK) return st;   // pos defaults to q_pos
  const Split sp_ws = attn_split(T, max_entries + window, H);
  const bool invariant = win_len != nullptr && g_batch_invariant.load(std::memory_order_relaxed) != 0;
  const Split sp_inv = attn_split_invariant(max_entries + window);
  const int n_need = invariant && sp_inv.n > sp_ws.n ? sp_inv.n : sp_ws.n;
  if ((st = check_ws(ws, ws_bytes, attn_partials_bytes(T, H, n_need, d), name)) != CSA_OK) return st;
  a.use_tc = attention_uses_tc(a);
  if ((st = need_tc_for_qrope(name, a)) != CSA_OK) return st;
  const Split sp = invariant ? sp_inv
                   : a.use_tc ? attn_split_tc(T, max_entries + window, H, sp_ws)
                   : a.d == 512 ? attn_split_512(T, max_entries + window, H, sp_ws) : sp_ws;
  a.n_split = sp.n;
  a.split_len = sp.len;
  a.err = static_cast<WsHeader*>(ws);
  if (sp.n > 1) {
    char* p = static_cast<char*>(ws) + kWsHeader;
    a.part_acc = reinterpret_cast<float*>(p);
    a.part_ml = reinterpret_cast<float*>(p + align256((size_t)T * sp.n * H * d * sizeof(float)));
  }
  Launch L{(cudaStream_t)stream};
  return cuda_status(launch_attention(L, a), name);
}

}  // extern "C"
