// Steps 2-3: lightning-indexer scoring and exact top-k selection.
//
// DeepSeek-V4 book, Ch.6 "How CSA Selects and Reads Memory": "The lightning
// indexer" (I[t,s] = sum_h w[t,h] ReLU(qI[t,h] . K[s]) over s < floor(t/m))
// and "Top-k selection and asymptotic scaling" (keep the k best entries).
//
// Scoring streams the indexer keys once (HBM-bound).  The grid is one resident
// wave: each CTA takes one chunk of one query's keys, its warps walk 16-key
// groups with four groups of 16-byte loads in flight per lane, and score them
// against all indexer heads with tensor-core mma (keys on M, heads on N, key
// dim as K).  The contraction dimension is permuted so that every lane reads whole
// 16-byte vectors of a key row: lane (g, q) loads dims [32v + 8q, 32v + 8q + 8)
// of rows g and g+8; the query fragments are loaded with the same
// permutation, which leaves every dot product unchanged.  Scores become
// order-preserving 32-bit keys.  In fused (few-query) mode only the keys that
// reach the query's threshold are appended to its candidate list (topk.cu
// finishes the selection); in many-query (prefill) mode every key is stored
// and a radix select per query, over its keys held in shared memory, picks
// the top k.
#include "kernels.h"
#include "score_mma.cuh"
#include "select.cuh"

namespace csa {

namespace {

// Tuning knobs (defaults measured on B200 with the 64-sequence, 128K-context
// decode workload).
#ifndef CSA_SCORE_UNROLL
#define CSA_SCORE_UNROLL 4
#endif
#ifndef CSA_SCORE_MINBLOCKS
#define CSA_SCORE_MINBLOCKS 3
#endif
constexpr int kScoreWarps = 8;
constexpr int kScoreThreads = kScoreWarps * 32;
constexpr int kUnroll = CSA_SCORE_UNROLL;   // 16-key groups in flight per warp

// One CTA scores a chunk of `chunk` keys of one query (the grid is sized by
// the host to one resident wave).  Each warp walks 16-key groups with
// kUnroll groups of loads in flight; keys are appended to the query's
// candidates (FUSED) or stored.
template <int CI, int NT, bool FUSED>
__global__ void __launch_bounds__(kScoreThreads, (CI == 64 && NT == 1) ? CSA_SCORE_MINBLOCKS : 1)
indexer_score_kernel(IndexerArgs a, int64_t chunk) {
  const int64_t tl = blockIdx.x;
  const int64_t t = a.t_begin + tl;
  const int64_t pos = a.q_pos ? __ldg(a.q_pos + t) : t;
  int64_t n_elig = pos / a.m;
  if (n_elig > a.max_entries) {
    if (blockIdx.y == 0 && threadIdx.x == 0) report(a.err, kErrEligible, (int32_t)t, n_elig);
    n_elig = a.max_entries;
  }
  if (FUSED && n_elig <= a.skip_le) return;
  const int64_t s_begin = (int64_t)blockIdx.y * chunk;
  if (s_begin >= n_elig) return;
  const int64_t s_end = min(s_begin + chunk, n_elig);
  const int32_t seq = a.seq_id ? __ldg(a.seq_id + t) : 0;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, q4 = lane & 3;
  QueryFrags<CI, NT> Q;
  Q.load(a, t, g, q4);
  const uint32_t tau = FUSED ? __ldg(a.tau + tl) : 0u;
  uint32_t* out = FUSED ? nullptr : a.keys_out + tl * a.key_stride;
  CandidateBatch<kUnroll> pend;   // the previous batch's candidates (fused mode)

  for (int64_t s0 = s_begin + (int64_t)warp * 16 * kUnroll; s0 < s_end;
       s0 += (int64_t)kScoreWarps * 16 * kUnroll) {
    uint4 kr[kUnroll][2][CI / 32];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t s = s0 + u * 16 + g + 8 * h;
        int64_t row = -1;
        if (s < s_end) row = cache_row(a.keys, seq, s, a.err, (int32_t)t);
#pragma unroll
        for (int v = 0; v < CI / 32; ++v)
          kr[u][h][v] = row >= 0 ? ld_stream_16(a.keys.data + row * CI + 32 * v + 8 * q4)
                                 : make_uint4(0, 0, 0, 0);
      }
    }
    bool pass[kUnroll];
    uint32_t keys[kUnroll], ents[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      float sg, s8;
      score_group<CI, NT>(kr[u], Q, sg, s8);
      const int64_t s = s0 + u * 16 + g + (q4 == 1 ? 8 : 0);
      const bool valid = q4 < 2 && s < s_end;
      keys[u] = score_key(q4 == 0 ? sg : s8);
      ents[u] = (uint32_t)s;
      pass[u] = valid && keys[u] >= tau;
      if (!FUSED && valid) out[s] = keys[u];
    }
    if (FUSED) {
      CandidateBatch<kUnroll> cur;
      cur.issue(a, tl, pass, keys, ents);
      pend.flush(a);
      pend = cur;
    }
  }
  if (FUSED) pend.flush(a);
}

constexpr int kSelThreads = 1024;
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_sums, int& total) {
  return sel::block_exclusive_scan<kSelThreads>(v, warp_sums, total);
}
__device__ __forceinline__ bool find_bin(const int* hist, int nbins, int need, int* warp_sums,
                                         uint32_t* s_bin, int* s_above, int* s_ok) {
  return sel::find_bin<kSelThreads>(hist, nbins, need, warp_sums, s_bin, s_above, s_ok);
}

// ---------------------------------------------------------------------------
// many-query (prefill) selection: radix select over keys in shared memory
// ---------------------------------------------------------------------------
constexpr int kBins = 2048;
constexpr int64_t kCommonPrefixMin = 8192;   // list length from which the common prefix is found first

__global__ void __launch_bounds__(kSelThreads) topk_select_radix_kernel(SelectArgs a) {
  extern __shared__ uint32_t skeys[];
  __shared__ int hist[kBins];
  __shared__ int warp_sums[32];
  __shared__ uint32_t s_bin;
  __shared__ int s_above, s_ok;

  const int64_t tl = blockIdx.x;
  const int64_t t = a.t_begin + tl;
  const int64_t pos = a.q_pos ? a.q_pos[t] : t;
  const int64_t n = min(pos / a.m, a.max_entries);
  const int k = a.top_k;
  int32_t* idx = a.idx_out + t * k;
  float* sco = a.score_out ? a.score_out + t * k : nullptr;
  const uint32_t* keys = a.keys + tl * a.key_stride;

  if (n <= k) {
    for (int64_t j = threadIdx.x; j < k; j += kSelThreads) {
      idx[j] = j < n ? (int32_t)j : -1;
      if (sco) sco[j] = j < n ? key_score(keys[j]) : -INFINITY;
    }
    if (threadIdx.x == 0) a.count_out[t] = (int32_t)n;
    return;
  }
  {
    // whole 16-byte vectors (rows are 256-byte aligned), several loads in flight
    const int64_t nv = (n + 3) >> 2;
    const uint4* kv = reinterpret_cast<const uint4*>(keys);
    uint4* sv = reinterpret_cast<uint4*>(skeys);
#pragma unroll 4
    for (int64_t v = threadIdx.x; v < nv; v += kSelThreads) sv[v] = kv[v];
  }
  __syncthreads();

  // the keys' common leading bits first (a min / max reduction), so that the
  // first radix digit spreads the keys instead of piling them into the few
  // bins of one exponent range; short lists skip it (it would cost more
  // than the atomics it saves)
  uint32_t kmin = 0u, kmax = 0xffffffffu;   // no common prefix assumed
  if (n >= kCommonPrefixMin) {                // uniform over the block
    kmin = 0xffffffffu;
    kmax = 0u;
    for (int64_t j = threadIdx.x; j < n; j += kSelThreads) {
      const uint32_t key = skeys[j];
      kmin = min(kmin, key);
      kmax = max(kmax, key);
    }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    __shared__ uint32_t s_min[32], s_max[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) {
      s_min[warp] = kmin;
      s_max[warp] = kmax;
    }
    __syncthreads();
    kmin = lane < kSelThreads / 32 ? s_min[lane] : 0xffffffffu;
    kmax = lane < kSelThreads / 32 ? s_max[lane] : 0u;
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
  }
  const int cpl = __clz(kmin ^ kmax);   // 32 when every key is equal
  uint32_t mask = cpl >= 32 ? 0xffffffffu : ~(0xffffffffu >> cpl);
  uint32_t prefix = kmin & mask;
  int remaining = k;
  int shift = 32 - cpl;   // bits below `shift` are still open
#pragma unroll 1
  while (shift > 0) {
    // an 11-bit digit; the last one is widened to 10 bits (find_bin takes
    // whole multiples of the block size), its upper bits then already fixed
    const int lo = shift > 11 ? shift - 11 : 0;
    const int dig = shift - lo >= 10 ? shift - lo : 10;
    const uint32_t dmask = (1u << dig) - 1u;
    for (int b = threadIdx.x; b < (1 << dig); b += kSelThreads) hist[b] = 0;
    __syncthreads();
    for (int64_t j = threadIdx.x; j < n; j += kSelThreads) {
      const uint32_t key = skeys[j];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> lo) & dmask], 1);
    }
    __syncthreads();
    find_bin(hist, 1 << dig, remaining, warp_sums, &s_bin, &s_above, &s_ok);
    prefix |= s_bin << lo;
    mask |= dmask << lo;
    remaining -= s_above;
    shift = lo;
    __syncthreads();
  }
  const uint32_t kth = prefix;

  int out_base = 0, tie_base = 0;
  for (int64_t base = 0; base < n; base += 4 * kSelThreads) {
    const int64_t j0 = base + 4 * threadIdx.x;
    uint32_t kk[4];
    int ties = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      kk[e] = j0 + e < n ? skeys[j0 + e] : 0u;
      ties += (j0 + e < n && kk[e] == kth);
    }
    int tie_total;
    int tie_rank = tie_base + block_exclusive_scan(ties, warp_sums, tie_total);
    bool sl[4];
    int nsel = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const bool valid = j0 + e < n;
      bool s = valid && kk[e] > kth;
      if (valid && kk[e] == kth) {
        s = tie_rank < remaining;
        ++tie_rank;
      }
      sl[e] = s;
      nsel += s;
    }
    int sel_total;
    int o = out_base + block_exclusive_scan(nsel, warp_sums, sel_total);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (sl[e] && o < k) {
        idx[o] = (int32_t)(j0 + e);
        if (sco) sco[o] = key_score(kk[e]);
        ++o;
      }
    }
    out_base += sel_total;
    tie_base += tie_total;
  }
  if (threadIdx.x == 0) a.count_out[t] = k;
}

template <int CI, int NT, bool FUSED>
cudaError_t launch_score(const Launch& L, const IndexerArgs& a, int64_t t_count) {
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, indexer_score_kernel<CI, NT, FUSED>,
                                                kScoreThreads, 0);
  if (per_sm < 1) per_sm = 1;
  // chunks per query so that the grid fills whole resident waves
  const int64_t wave = (int64_t)sms * per_sm;
  int64_t per_q = wave / t_count;
  if (per_q < 1) per_q = 1;
  const int64_t min_chunk = 16 * kScoreWarps * kUnroll;     // one pass of the warps
  int64_t chunk = (a.max_entries + per_q - 1) / per_q;
  chunk = (chunk + min_chunk - 1) / min_chunk * min_chunk;
  if (chunk < min_chunk) chunk = min_chunk;
  per_q = (a.max_entries + chunk - 1) / chunk;
  const dim3 grid((unsigned)t_count, (unsigned)per_q);
  prefer_max_shared(indexer_score_kernel<CI, NT, FUSED>);
  indexer_score_kernel<CI, NT, FUSED><<<grid, kScoreThreads, 0, L.stream>>>(a, chunk);
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_indexer_scores(const Launch& L, const IndexerArgs& a, int64_t t_count) {
  if (t_count == 0 || a.max_entries == 0) return cudaSuccess;
  if (a.fp4) return launch_indexer_scores_fp4(L, a, t_count);
#ifndef CSA_NO_TC_INDEXER
  if (tc_indexer_prefill_supported(a, t_count)) return launch_indexer_scores_tc_prefill(L, a, t_count, false);
  if (tc_indexer_supported(a, t_count)) return launch_indexer_scores_tc(L, a, t_count);
#endif
  const int nt = (a.H_I + 7) / 8;
  const int ntb = nt <= 1 ? 1 : nt <= 2 ? 2 : nt <= 4 ? 4 : 8;
  const bool fused = a.tau != nullptr;
  L.begin(kKernelIndexerScore);
#define CSA_SCORE_CASE(CI_, NT_)                                                        \
  if (a.c_I == CI_ && ntb == NT_) {                                                     \
    if (fused) launch_score<CI_, NT_, true>(L, a, t_count);                     \
    else launch_score<CI_, NT_, false>(L, a, t_count);                          \
  }
  CSA_SCORE_CASE(64, 1)
  CSA_SCORE_CASE(64, 2)
  CSA_SCORE_CASE(64, 4)
  CSA_SCORE_CASE(64, 8)
  CSA_SCORE_CASE(128, 1)
  CSA_SCORE_CASE(128, 2)
  CSA_SCORE_CASE(128, 4)
  CSA_SCORE_CASE(128, 8)
#undef CSA_SCORE_CASE
  return L.end(kKernelIndexerScore);
}

cudaError_t launch_topk_select(const Launch& L, const SelectArgs& a, int64_t t_count) {
  if (t_count == 0) return cudaSuccess;
  L.begin(kKernelTopkSelect);
  const size_t bytes = (size_t)((a.max_entries + 3) & ~int64_t(3)) * sizeof(uint32_t);   // whole uint4 stores
  prefer_max_shared(topk_select_radix_kernel);
  cudaFuncSetAttribute(topk_select_radix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       kRadixSelectMaxEntries * (int)sizeof(uint32_t));
  topk_select_radix_kernel<<<(unsigned)t_count, kSelThreads, bytes, L.stream>>>(a);
  return L.end(kKernelTopkSelect);
}

}  // namespace csa
