// Step 2 on the CUDA-core tensor path (mma.sync): lightning-indexer scoring
// for the shapes the tcgen05 scorers do not take (c_I = 128, other H_I, many
// queries on several sequences).
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
// order-preserving 32-bit keys; only the keys that reach the query's
// threshold are appended to its candidate list (topk.cu samples the threshold
// and finishes the selection).
#include "kernels.h"
#include "score_mma.cuh"

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
// kUnroll groups of loads in flight; keys that reach the query's threshold
// are appended to its candidates.
template <int CI, int NT>
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
  if (n_elig <= a.skip_le) return;
  const int64_t s_begin = (int64_t)blockIdx.y * chunk;
  if (s_begin >= n_elig) return;
  const int64_t s_end = min(s_begin + chunk, n_elig);
  const int32_t seq = a.seq_id ? __ldg(a.seq_id + t) : 0;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, q4 = lane & 3;
  QueryFrags<CI, NT> Q;
  Q.load(a, t, g, q4);
  const uint32_t tau = __ldg(a.tau + tl);
  CandidateBatch<kUnroll> pend;   // the previous batch's candidates

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
    }
    CandidateBatch<kUnroll> cur;
    cur.issue(a, tl, pass, keys, ents);
    pend.flush(a);
    pend = cur;
  }
  pend.flush(a);
}

template <int CI, int NT>
cudaError_t launch_score(const Launch& L, const IndexerArgs& a, int64_t t_count) {
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, indexer_score_kernel<CI, NT>,
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
  prefer_max_shared(indexer_score_kernel<CI, NT>);
  indexer_score_kernel<CI, NT><<<grid, kScoreThreads, 0, L.stream>>>(a, chunk);
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
  L.begin(kKernelIndexerScore);
#define CSA_SCORE_CASE(CI_, NT_) \
  if (a.c_I == CI_ && ntb == NT_) launch_score<CI_, NT_>(L, a, t_count);
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

}  // namespace csa
