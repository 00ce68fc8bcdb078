// Steps 2-3: lightning-indexer scoring and exact top-k selection.
//
// DeepSeek-V4 book, Ch.6 "How CSA Selects and Reads Memory": "The lightning
// indexer" (I[t,s] = sum_h w[t,h] ReLU(qI[t,h] . K[s]) over s < floor(t/m))
// and "Top-k selection and asymptotic scaling" (keep the k best entries).
//
// Scoring streams the indexer keys once.  Each warp takes 16 keys at a time
// and scores them against all indexer heads with tensor-core mma (keys on M,
// heads on N, key dim as K).  The contraction dimension is permuted so that
// every lane reads whole 16-byte vectors of a key row: lane (g, q) loads dims
// [32v + 8q, 32v + 8q + 8) of rows g and g+8; the query fragments are loaded
// with the same permutation, which leaves every dot product unchanged.
//
// Selection is an exact radix select on order-preserving 32-bit keys of the
// fp32 scores (11 + 11 + 10 bits), then an index-ordered compaction: entries
// above the k-th key, plus the lowest-index entries equal to it.  The output
// is therefore ascending and independent of thread scheduling.
#include "kernels.h"

namespace csa {

namespace {

constexpr int kScoreWarps = 8;
constexpr int kScoreChunk = 2048;      // entries per CTA
constexpr int kUnroll = 2;             // 16-row groups in flight per warp

template <int CI, int NT>
__global__ void __launch_bounds__(kScoreWarps * 32) indexer_score_kernel(IndexerArgs a) {
  constexpr int NV = CI / 32;   // 16-byte vectors per row per lane
  constexpr int KS = CI / 16;   // mma k-steps
  const int64_t t = a.t_begin + blockIdx.x;
  const int64_t pos = a.q_pos ? __ldg(a.q_pos + t) : t;
  int64_t n_elig = pos / a.m;
  if (n_elig > a.max_entries) {
    if (blockIdx.y == 0 && threadIdx.x == 0) report(a.err, kErrEligible, (int32_t)t, n_elig);
    n_elig = a.max_entries;
  }
  const int64_t s_begin = (int64_t)blockIdx.y * kScoreChunk;
  if (s_begin >= n_elig) return;
  const int64_t s_end = min(s_begin + kScoreChunk, n_elig);
  const int32_t seq = a.seq_id ? __ldg(a.seq_id + t) : 0;

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, q4 = lane & 3;

  // query fragments (B operand, col-major): head n = nt*8 + g
  uint32_t bq[NT][KS][2];
  float wv[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int head = nt * 8 + g;
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      uint4 u = make_uint4(0, 0, 0, 0);
      if (head < a.H_I)
        u = __ldg(reinterpret_cast<const uint4*>(a.q_idx + ((t * a.H_I + head) * CI) + 32 * v +
                                                 8 * q4));
      bq[nt][2 * v][0] = u.x;
      bq[nt][2 * v][1] = u.y;
      bq[nt][2 * v + 1][0] = u.z;
      bq[nt][2 * v + 1][1] = u.w;
    }
    const int h0 = nt * 8 + 2 * q4;
    wv[nt][0] = h0 < a.H_I ? __ldg(a.w + t * a.H_I + h0) : 0.f;
    wv[nt][1] = h0 + 1 < a.H_I ? __ldg(a.w + t * a.H_I + h0 + 1) : 0.f;
  }

  const __nv_bfloat16* kbase = a.keys.data;
  float* out = a.scores + (t - a.t_begin) * a.score_stride;

  for (int64_t s0 = s_begin + (int64_t)warp * 16 * kUnroll; s0 < s_end;
       s0 += (int64_t)kScoreWarps * 16 * kUnroll) {
    uint4 kr[kUnroll][2][NV];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t s = s0 + u * 16 + g + 8 * h;
        int64_t row = -1;
        if (s < s_end) row = cache_row(a.keys, seq, s, a.err, (int32_t)t);
#pragma unroll
        for (int v = 0; v < NV; ++v)
          kr[u][h][v] = row >= 0 ? ld_stream_16(kbase + row * CI + 32 * v + 8 * q4)
                                 : make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      float sg = 0.f, s8 = 0.f;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int v = 0; v < NV; ++v) {
          const uint32_t lo[4] = {kr[u][0][v].x, kr[u][1][v].x, kr[u][0][v].y, kr[u][1][v].y};
          mma_bf16_16816(d, lo, bq[nt][2 * v][0], bq[nt][2 * v][1]);
          const uint32_t hi[4] = {kr[u][0][v].z, kr[u][1][v].z, kr[u][0][v].w, kr[u][1][v].w};
          mma_bf16_16816(d, hi, bq[nt][2 * v + 1][0], bq[nt][2 * v + 1][1]);
        }
        sg = fmaf(wv[nt][0], fmaxf(d[0], 0.f), sg);
        sg = fmaf(wv[nt][1], fmaxf(d[1], 0.f), sg);
        s8 = fmaf(wv[nt][0], fmaxf(d[2], 0.f), s8);
        s8 = fmaf(wv[nt][1], fmaxf(d[3], 0.f), s8);
      }
      sg += __shfl_xor_sync(0xffffffffu, sg, 1);
      s8 += __shfl_xor_sync(0xffffffffu, s8, 1);
      sg += __shfl_xor_sync(0xffffffffu, sg, 2);
      s8 += __shfl_xor_sync(0xffffffffu, s8, 2);
      const int64_t s = s0 + u * 16 + g + (q4 == 1 ? 8 : 0);
      if (q4 < 2 && s < s_end) out[s] = q4 == 0 ? sg : s8;
    }
  }
}

// ---------------------------------------------------------------------------
// top-k selection: one 1024-thread CTA per query
// ---------------------------------------------------------------------------
constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kBins = 2048;
constexpr int kSmemKeyCap = 48 * 1024;   // keys held in shared memory (192 KB)

// Block-wide exclusive scan of one int per thread; returns the block total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_sums, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int s = lane < kSelWarps ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    warp_sums[lane] = s;   // inclusive prefix of warp totals
  }
  __syncthreads();
  total = warp_sums[kSelWarps - 1];
  const int base = warp ? warp_sums[warp - 1] : 0;
  __syncthreads();   // warp_sums is reused by the next scan
  return base + x - v;
}

template <bool SMEM>
__global__ void __launch_bounds__(kSelThreads) topk_select_kernel(SelectArgs a) {
  extern __shared__ uint32_t skeys[];
  __shared__ int hist[kBins];
  __shared__ int warp_sums[32];
  __shared__ uint32_t s_bin;
  __shared__ int s_above;

  const int64_t t = a.t_begin + blockIdx.x;
  const int64_t pos = a.q_pos ? a.q_pos[t] : t;
  const int64_t n = min(pos / a.m, a.max_entries);
  const int k = a.top_k;
  int32_t* idx = a.idx_out + t * k;
  float* sco = a.score_out ? a.score_out + t * k : nullptr;
  const float* sc = a.scores + (t - a.t_begin) * a.score_stride;

  if (n <= k) {   // everything eligible is selected
    for (int64_t j = threadIdx.x; j < k; j += kSelThreads) {
      idx[j] = j < n ? (int32_t)j : -1;
      if (sco) sco[j] = j < n ? sc[j] : -INFINITY;
    }
    if (threadIdx.x == 0) a.count_out[t] = (int32_t)n;
    return;
  }

  if (SMEM) {
    for (int64_t j = threadIdx.x; j < n; j += kSelThreads) skeys[j] = score_key(sc[j]);
    __syncthreads();
  }
  auto key_of = [&](int64_t j) -> uint32_t { return SMEM ? skeys[j] : score_key(sc[j]); };

  // radix select of the k-th largest key: digits of 11, 11 and 10 bits
  uint32_t prefix = 0, mask = 0;
  int remaining = k;
  const int shifts[3] = {21, 10, 0};
  const uint32_t digit_mask[3] = {0x7ffu, 0x7ffu, 0x3ffu};
#pragma unroll 1
  for (int p = 0; p < 3; ++p) {
    for (int b = threadIdx.x; b < kBins; b += kSelThreads) hist[b] = 0;
    __syncthreads();
    for (int64_t j = threadIdx.x; j < n; j += kSelThreads) {
      const uint32_t key = key_of(j);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shifts[p]) & digit_mask[p]], 1);
    }
    __syncthreads();
    // suffix counts over bins (from the top): thread handles bins 2t', 2t'+1
    // in descending order (rank r = kBins-1-bin)
    const int r0 = 2 * threadIdx.x;
    const int c0 = hist[kBins - 1 - r0], c1 = hist[kBins - 2 - r0];
    int tot;
    const int before = block_exclusive_scan(c0 + c1, warp_sums, tot);
    // bins above (kBins-1-r0) hold `before` keys
    if (before < remaining && before + c0 >= remaining) {
      s_bin = kBins - 1 - r0;
      s_above = before;
    } else if (before + c0 < remaining && before + c0 + c1 >= remaining) {
      s_bin = kBins - 2 - r0;
      s_above = before + c0;
    }
    __syncthreads();
    prefix |= s_bin << shifts[p];
    mask |= digit_mask[p] << shifts[p];
    remaining -= s_above;
    __syncthreads();
  }
  const uint32_t kth = prefix;   // the k-th largest key; take `remaining` of its ties

  // index-ordered compaction, 4 consecutive entries per thread per tile
  int out_base = 0, tie_base = 0;
  for (int64_t base = 0; base < n; base += 4 * kSelThreads) {
    const int64_t j0 = base + 4 * threadIdx.x;
    uint32_t kk[4];
    int ties = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      kk[e] = j0 + e < n ? key_of(j0 + e) : 0u;
      ties += (j0 + e < n && kk[e] == kth);
    }
    int tie_total;
    int tie_rank = tie_base + block_exclusive_scan(ties, warp_sums, tie_total);
    bool sel[4];
    int nsel = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const bool valid = j0 + e < n;
      bool s = valid && kk[e] > kth;
      if (valid && kk[e] == kth) {
        s = tie_rank < remaining;
        ++tie_rank;
      }
      sel[e] = s;
      nsel += s;
    }
    int sel_total;
    int o = out_base + block_exclusive_scan(nsel, warp_sums, sel_total);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (sel[e] && o < k) {
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

}  // namespace

cudaError_t launch_indexer_scores(const Launch& L, const IndexerArgs& a, int64_t t_count) {
  if (t_count == 0 || a.max_entries == 0) return cudaSuccess;
  const dim3 grid((unsigned)t_count, (unsigned)((a.max_entries + kScoreChunk - 1) / kScoreChunk));
  const int nt = (a.H_I + 7) / 8;
  L.begin(kKernelIndexerScore);
#define CSA_SCORE_CASE(CI_, NT_)                                                   \
  if (a.c_I == CI_ && nt == NT_) {                                                 \
    indexer_score_kernel<CI_, NT_><<<grid, kScoreWarps * 32, 0, L.stream>>>(a);    \
    return L.end(kKernelIndexerScore);                                             \
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
  // 3, 5, 6, 7 n-tiles round up to the next built variant
  if (a.c_I == 64) {
    if (nt <= 4) indexer_score_kernel<64, 4><<<grid, kScoreWarps * 32, 0, L.stream>>>(a);
    else indexer_score_kernel<64, 8><<<grid, kScoreWarps * 32, 0, L.stream>>>(a);
  } else {
    if (nt <= 4) indexer_score_kernel<128, 4><<<grid, kScoreWarps * 32, 0, L.stream>>>(a);
    else indexer_score_kernel<128, 8><<<grid, kScoreWarps * 32, 0, L.stream>>>(a);
  }
  return L.end(kKernelIndexerScore);
}

cudaError_t launch_topk_select(const Launch& L, const SelectArgs& a, int64_t t_count) {
  if (t_count == 0) return cudaSuccess;
  const bool smem = a.max_entries <= kSmemKeyCap;
  L.begin(kKernelTopkSelect);
  if (smem) {
    const size_t bytes = (size_t)a.max_entries * sizeof(uint32_t);
    cudaFuncSetAttribute(topk_select_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kSmemKeyCap * (int)sizeof(uint32_t));
    topk_select_kernel<true><<<(unsigned)t_count, kSelThreads, bytes, L.stream>>>(a);
  } else {
    topk_select_kernel<false><<<(unsigned)t_count, kSelThreads, 0, L.stream>>>(a);
  }
  return L.end(kKernelTopkSelect);
}

}  // namespace csa
