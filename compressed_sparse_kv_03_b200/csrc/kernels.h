// Internal launch interface between the C-ABI layer (api.cu) and the kernels.
#pragma once

#include <utility>

#include "common.cuh"

namespace csa {

enum KernelId : int32_t {
  kKernelIndexerScore = 0,
  kKernelTopkSelect = 1,
  kKernelAttention = 2,
  kKernelMerge = 3,
  kKernelCompress = 4,
  kKernelQuantize = 5,
  kKernelTopkSample = 6,   // the fused selection's sampling / threshold pass
  kNumKernelIds = 7,
};

// Per-call launch context: the stream plus the timing / launch-count hooks.
struct Launch {
  cudaStream_t stream;
  void begin(int32_t kernel) const;              // records the kernel's begin event, if attached
  cudaError_t end(int32_t kernel) const;         // counts the launch, records the end event, checks
};

cudaError_t launch_compress(const Launch& L, const __nv_bfloat16* Ca, const __nv_bfloat16* Za,
                            const __nv_bfloat16* Cb, const __nv_bfloat16* Zb, const float* bias,
                            int64_t n_tokens, int dim, int m, int overlap, __nv_bfloat16* out);

// Decode-time cache append (one token per sequence): see cache.cu.
struct CacheAppendArgs {
  const __nv_bfloat16 *Ca, *Za, *Cb, *Zb;   // [B, dim] the new tokens (Cb / Zb null: Ca / Za)
  const float* bias;                         // [m, dim] or [2, m, dim] or null
  const int64_t* pos;                        // [B] position t of each new token
  int B, dim, m, overlap;
  __nv_bfloat16 *blk_c, *blk_z;              // [B, m, dim] the unfinished block's a-branch rows
  __nv_bfloat16 *bb_c, *bb_z;                // [B, 2, m, dim] b-branch rows by block parity (overlap)
  __nv_bfloat16* win;                        // [B, window, dim] ring of raw rows, slot t mod window
  int window;
  CacheRef cache;                            // compressed entries, written at entry t / m
  int64_t max_entries;
  WsHeader* err;
};
cudaError_t launch_cache_append(const Launch& L, const CacheAppendArgs& a);

// RMSNorm (eps >= 0) and / or partial RoPE (rope_dims > 0) of [T, H, dim]
// vectors: see normrope.cu.
struct NormRopeArgs {
  const __nv_bfloat16* x;
  __nv_bfloat16* out;                        // may equal x
  int64_t T;
  int H, dim;
  const float* gain;                         // [dim] or null
  float eps;                                 // < 0: no RMSNorm
  const int64_t* pos;                        // [T] or null (row index)
  int64_t pos_mul;                           // position = (pos ? pos[t] : t) * pos_mul
  int rope_dims;                             // rotated trailing coordinates (0: none)
  float rope_base;
  int inverse;                               // 1: R_{-t}
  double theta[128];                         // pair frequencies base^(-2j / rope_dims) (host-filled)
};
cudaError_t launch_norm_rope(const Launch& L, const NormRopeArgs& a);

// Indexer selection: the scorer keeps only the (key, entry) pairs that reach
// a per-query threshold drawn from a sample of the query's scores, and a
// finishing pass selects exactly among them (no score matrix is stored).
// Few-query (decode) mode, at most kFusedMaxQueries queries per launch: a
// per-query sample launch and one CTA per query to finish.  Many-query mode
// (more queries per call, at most kManyMaxEntries entries each): the tcgen05
// scorer samples its own keys, and one warp per query sets the threshold and
// finishes (its selection bitmaps bound the entries per query).
constexpr int64_t kMaxSelectEntries = int64_t(1) << 19;
constexpr int64_t kFusedMaxQueries = 2048;
constexpr int64_t kManyMaxEntries = 48 * 1024;

// Lightning-indexer scores of every eligible entry for every query of one
// chunk of queries: the entries whose order-preserving key reaches
// tau[t - t_begin] are appended to the query's candidate list.
struct IndexerArgs {
  const __nv_bfloat16* q_idx;   // [T, H_I, c_I]
  const float* w;               // [T, H_I]
  CacheRef keys;
  const int32_t* seq_id;        // [T] or null
  const int64_t* q_pos;         // [T] or null
  int64_t T;
  int H_I, c_I, m;
  int64_t max_entries;
  int64_t t_begin;              // first query of this launch (chunking)
  uint32_t* work;               // zeroed work counter of the tcgen05 scorer
  // selection
  const uint32_t* tau = nullptr;     // [T_chunk] candidate threshold (a score key)
  uint32_t* cand_count = nullptr;    // [T_chunk] zeroed; counts every pair that passes
  uint2* cand = nullptr;             // [T_chunk, cand_cap] (key, entry), first cand_cap kept
  int64_t cand_cap = 0;
  int64_t skip_le = 0;               // queries with at most this many eligible entries are
                                     // not scored (they select all of them)
  // many-query (prefill) selection: the tcgen05 scorer's sample pass writes
  // each query's sampled keys here ([T_chunk, kPSampleKeys]); queries whose
  // candidate count misses [top_k, cand_cap] are listed for the exact fallback
  uint32_t* psample = nullptr;
  // tcgen05 4-bit scorer: per chunk query, its quantized heads as the MMA's B
  // operand image (written by launch_fp4_query_images, read by both passes)
  uint8_t* q_img = nullptr;
  uint32_t* fb_list = nullptr;       // [T_chunk] chunk-local query ids
  uint32_t* fb_count = nullptr;      // zeroed by the threshold pass
  WsHeader* err;
  // 4-bit mode (fp4 = 1): q_idx is quantized to E2M1 codes + scale bytes in
  // the scorer; keys.data holds rows of c_I/2 code bytes and k_scales rows of
  // c_I/32 scale bytes at the same physical row index
  int fp4 = 0;
  const uint8_t* k_scales = nullptr;
};
cudaError_t launch_indexer_scores(const Launch& L, const IndexerArgs& a, int64_t t_count);

// Many-query sampling: a block of 128 / H_I consecutive queries (the tcgen05
// scorer's block) shares kPSampleChunks whole 256-key chunks spread evenly
// over the entries every query of the block can read; a query's sample is
// those chunks' keys.  Blocks whose queries all keep every key as a candidate
// (2 n <= cand_cap) or select every entry (n <= skip_le) take no sample.
constexpr int kPSampleChunks = 4;
constexpr int kPSampleKeys = kPSampleChunks * 256;
__host__ __device__ inline int psample_chunks(int64_t nmin, int64_t nmax, int64_t cand_cap,
                                              int64_t skip_le) {
  if (nmax <= skip_le || 2 * nmax <= cand_cap) return 0;
  const int64_t c = nmin / 256;
  return c < kPSampleChunks ? (int)c : kPSampleChunks;
}
// The i-th of sc sampled chunks of a block whose queries all read nmin entries.
__host__ __device__ inline int64_t psample_chunk(int i, int sc, int64_t nmin) {
  return ((2 * (int64_t)i + 1) * (nmin / 256)) / (2 * (int64_t)sc);
}
// Fused-selection epilogue of the scorers, one warp at a time: a batch of U
// keys per lane (entry ids alongside) whose `pass` flags mark the candidates.
// issue() takes the warp's ballots and reserves slots with one atomic on the
// query's count; flush() stores the batch into the reserved slots.  A scorer
// issues batch j and flushes batch j-1 after it, so the atomic's round trip
// overlaps the next batch instead of stalling the warp.  Slots past cand_cap
// are counted but not stored.  Every lane of the warp must make each call.
template <int U>
struct CandidateBatch {
  uint32_t key[U], ent[U], m[U];
  uint32_t base = 0, tot = 0;
  int64_t tl = 0;
  __device__ __forceinline__ void issue(const IndexerArgs& a, int64_t tl_, const bool (&pass)[U],
                                        const uint32_t (&k)[U], const uint32_t (&e)[U]) {
    uint32_t t = 0;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      m[u] = __ballot_sync(0xffffffffu, pass[u]);
      key[u] = k[u];
      ent[u] = e[u];
      t += (uint32_t)__popc(m[u]);
    }
    tot = t;
    tl = tl_;
    if (t != 0u && (threadIdx.x & 31) == 0) base = atomicAdd(a.cand_count + tl_, t);
  }
  __device__ __forceinline__ void flush(const IndexerArgs& a) {
    if (tot == 0u) return;   // warp-uniform
    const int lane = threadIdx.x & 31;
    uint32_t off = __shfl_sync(0xffffffffu, base, 0);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if ((m[u] >> lane) & 1u) {
        const uint32_t slot = off + (uint32_t)__popc(m[u] & ((1u << lane) - 1u));
        if (slot < (uint64_t)a.cand_cap) a.cand[tl * a.cand_cap + slot] = make_uint2(key[u], ent[u]);
      }
      off += (uint32_t)__popc(m[u]);
    }
    tot = 0u;
  }
};

// tcgen05 + TMA scoring path (c_I = 64, H_I <= 16, pages a multiple of 64 rows;
// fused mode only)
bool tc_indexer_supported(const IndexerArgs& a, int64_t t_count);
cudaError_t launch_indexer_scores_tc(const Launch& L, const IndexerArgs& a, int64_t t_count);
// tcgen05 many-query path: all queries on one sequence (seq_id null), c_I = 64,
// H_I in {4, 8, 16}; blocks of 128 / H_I queries share each key tile.  Its
// sample pass (sample = true) writes a.psample, its fused pass candidates.
bool tc_indexer_prefill_supported(const IndexerArgs& a, int64_t t_count);
cudaError_t launch_indexer_scores_tc_prefill(const Launch& L, const IndexerArgs& a, int64_t t_count,
                                             bool sample);
// tcgen05 4-bit scorer (few-query mode, c_I in {64, 128}, H_I <= 64, pages a
// multiple of 64 rows): block-scaled MMAs on the stored codes; its sample pass
// (sample = true) writes a.psample for topk_threshold_many, its fused pass the
// candidate lists
bool tc_fp4_indexer_supported(const IndexerArgs& a, int64_t t_count);
cudaError_t launch_indexer_scores_fp4_tc(const Launch& L, const IndexerArgs& a, int64_t t_count, bool sample);
// Quantizes each chunk query's heads into its operand image at a.q_img (at
// most kFp4ImgSlots * 8 bytes per query) and zeroes the work counter; runs
// before the tcgen05 4-bit scorer's passes.
constexpr int kFp4ImgSlots = 640;
cudaError_t launch_fp4_query_images(const Launch& L, const IndexerArgs& a, int64_t t_count);
// 4-bit scorer (E2M1 codes with one scale byte per 32 elements): see indexer_fp4.cu
cudaError_t launch_indexer_scores_fp4(const Launch& L, const IndexerArgs& a, int64_t t_count);
// [n_blocks * 32] bf16 -> n_blocks * 16 code bytes + n_blocks scale bytes
cudaError_t launch_mxfp4_quantize(const Launch& L, const __nv_bfloat16* x, int64_t n_blocks,
                                  uint8_t* codes, uint8_t* scales);


// Few-query selection, around the scoring launch of the same
// IndexerArgs (tau / cand_count / cand / cand_cap / skip_le / work set):
//   launch_topk_sample: per query, zeroes its candidate count (and the work
//     counter), scores a strided sample of its eligible entries and writes a
//     threshold tau that about 2 top_k of its entries are expected to reach;
//   launch_topk_finish: per query, the exact top-k -- among the candidates when
//     top_k <= count <= cand_cap, else by exact recompute passes over every
//     eligible entry -- written ascending with its count (and scores).
cudaError_t launch_topk_sample(const Launch& L, const IndexerArgs& a, int top_k, int64_t t_count);
cudaError_t launch_topk_finish(const Launch& L, const IndexerArgs& a, int top_k, int32_t* idx_out,
                               int32_t* count_out, float* score_out, int64_t t_count);
// Many-query (prefill) selection, one warp per query, after the tcgen05
// scorer's sample pass and around its fused pass (fb_list / fb_count /
// psample set):
//   launch_topk_threshold_many: tau from the sampled keys (the sample of a block
//     of qb consecutive queries: 128 / H_I for the prefill scorer, 1 for the
//     4-bit decode scorer); zeroes the counts, the fallback list and the work
//     counter;
//   launch_topk_finish_many: the exact top-k among the candidates, then the
//     recompute of the listed queries whose count missed [top_k, cand_cap].
bool topk_many_supported(const IndexerArgs& a);
cudaError_t launch_topk_threshold_many(const Launch& L, const IndexerArgs& a, int top_k, int64_t t_count,
                                      int qb);
cudaError_t launch_topk_finish_many(const Launch& L, const IndexerArgs& a, int top_k, int32_t* idx_out,
                                    int32_t* count_out, float* score_out, int64_t t_count);

// Attention over a virtual row list per query: its selected / eligible
// compressed entries followed by its window rows.
struct AttnArgs {
  int d = 128;                  // head dim: 128, or 512 (attention512.cu, mma.sync only)
  const __nv_bfloat16* q;       // [T, H, d]
  int64_t T;
  int H;
  CacheRef kv;                  // compressed entries
  int seq_per_query;            // 1: query i reads sequence i; 0: all read sequence 0
  const int32_t* seq_id = nullptr;   // [T]: query i reads sequence seq_id[i] (overrides
                                     // seq_per_query); without win_len the raw rows are
                                     // packed: query i is raw row i of `win`
  // entry list: explicit (idx != null) or all s < floor(pos/m)
  const int32_t* idx;
  int top_k;
  const int32_t* count;
  const int64_t* q_pos;         // null: query i at position i
  int m;
  int64_t max_entries;
  // window: buffer [T, window, 128] with win_len (decode) or raw rows (win_len null)
  const __nv_bfloat16* win;
  const int32_t* win_len;
  int window;
  int64_t win_rows;             // raw rows of `win` when win_len is null (0 = unknown)
  float sm_scale;
  const float* sink;            // [H] or null
  __nv_bfloat16* out;           // [T, H, 128]
  float* lse;                   // [T, H] or null
  // split-KV
  int n_split;
  int split_len;                // rows of the virtual list per split (multiple of 64)
  float* part_acc;              // [T, n_split, H, 128]
  float* part_ml;               // [T, n_split, H, 2]
  WsHeader* err;
  int use_tc;                   // tcgen05 kernel (else mma.sync); see attention_uses_tc
  // mixed-precision entries (kv_fp8 = 1, mma.sync kernel only): kv.data holds
  // rows of 128 - rope_dims E4M3 codes, kv_scales rows of (128 - rope_dims)/32
  // scale bytes and kv_rope rows of rope_dims bf16, all at the entry's
  // physical row; window rows stay bf16
  int kv_fp8 = 0;
  const uint8_t* kv_scales = nullptr;
  const __nv_bfloat16* kv_rope = nullptr;
  int rope_dims = 0;
  // query prologue / output epilogue (tcgen05 kernel only): RMSNorm of every
  // query head (q_norm_eps >= 0, gain q_norm_gain [128] or null), rotation of
  // its last q_rope_dims coordinates by R_t, and with out_derotate the
  // output's by R_{-t}; t = rope_pos[i] (or q_pos[i], or i)
  int qprologue = 0;
  const float* q_norm_gain = nullptr;
  float q_norm_eps = -1.f;
  int q_rope_dims = 0;
  float q_rope_base = 10000.f;
  int out_derotate = 0;
  const int64_t* rope_pos = nullptr;
  // cycles a pipeline wait of the tcgen05 kernel may take before it gives up
  // and records a timeout; withhold_q (failure-detection self-test) skips the
  // first work item's query-tile copy so that those waits run out
  long long wait_limit = 2000000000ll;
  int withhold_q = 0;
};
cudaError_t launch_attention(const Launch& L, const AttnArgs& a);

// Sequence whose compressed entries query i reads.
__device__ __forceinline__ int32_t attn_seq(const AttnArgs& a, int64_t i) {
  return a.seq_id ? __ldg(a.seq_id + i) : (a.seq_per_query ? (int32_t)i : 0);
}

// Window of query i at position pos when the window comes from raw rows
// (win_len null): n_win = min(pos + 1, window) rows ending at the query's own
// raw row -- row pos of `win`, or row i when the rows are packed (seq_id
// given).  A packed row list that would start before row 0 is cut there and
// reported (kErrWindow).  Returns the first row; sets n_win.
__device__ __forceinline__ int64_t attn_raw_window(const AttnArgs& a, int64_t i, int64_t pos,
                                                   int64_t& n_win, bool do_report) {
  n_win = pos + 1 < a.window ? pos + 1 : a.window;
  const int64_t last = a.seq_id ? i : pos;
  if (last - n_win + 1 < 0) {
    if (do_report) report(a.err, kErrWindow, (int32_t)i, pos);
    n_win = last + 1;
  }
  return last - n_win + 1;
}
// tcgen05 path (d = 128; any H, in groups of 64 heads)
bool tc_attention_supported(const AttnArgs& a);
// 0 automatic, 1 tensor-core kernel, 2 mma.sync kernel
int32_t attention_kernel_choice();
// true once after csa_test_attention_timeout(1): the next tensor-core
// attention launch runs the self-test
bool take_attention_timeout_test();
// Which attention kernel a call with these arguments runs (fields other than
// the split / workspace ones must be set).
bool attention_uses_tc(const AttnArgs& a);
cudaError_t launch_attention_tc(const Launch& L, const AttnArgs& a);
// head dim 512: one CTA per (query, slice, 16 heads), warps split the dims
cudaError_t launch_attention512(const Launch& L, const AttnArgs& a);

// [n, dim] bf16 entries -> E4M3 codes [n, dim - rope] + scale bytes
// [n, (dim - rope)/32] + rotary part [n, rope] bf16: see fp8_entry.cu
cudaError_t launch_fp8_entry_quantize(const Launch& L, const __nv_bfloat16* x, int64_t n, int dim,
                                      int rope, uint8_t* codes, uint8_t* scales,
                                      __nv_bfloat16* rope_out);

// Every kernel asks for the largest shared-memory carveout, so that the
// kernels of a step, some of which need nearly all of it, never make the SMs
// repartition L1 and shared memory between launches.
template <class K>
inline void prefer_max_shared(K kernel) {
  cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                       (int)cudaSharedmemCarveoutMaxShared);
}

// Launch `kernel`, with programmatic stream serialization when `pdl` (the
// kernel then must call pdl_wait() before it reads anything a predecessor
// writes).
template <class... P, class... A>
inline cudaError_t launch_kernel(void (*kernel)(P...), dim3 grid, dim3 block, size_t smem,
                                 cudaStream_t stream, bool pdl, A&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  if (pdl) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
}

// Text returned by csa_last_error() for this thread.
void set_last_error(const char* msg);

// Host-side argument checks of csa_sparse_attn_decode (B > 0): CSA_OK or the
// status and message that call would return, with nothing enqueued.
csa_status_t check_decode_call(const char* name, const csa_bf16* q, const csa_cache_t* kv,
                               const csa_bf16* win, const int32_t* win_len, const int32_t* idx,
                               const int32_t* count, int32_t B, int32_t H, int32_t d,
                               int32_t top_k, int32_t window, const csa_bf16* out);

}  // namespace csa
