// Step 3 fused with step 2: exact top-k without a stored score matrix.
//
// DeepSeek-V4 book, Ch.6 "The lightning indexer" (scores I[t,s] = sum_h
// w[t,h] ReLU(qI[t,h] . K[s]) over s < floor(t/m)) and "Top-k selection and
// asymptotic scaling" (keep the k best entries).
//
// Three launches per chunk of queries:
// Consecutive launches overlap (programmatic dependent launch): the scorer
// starts streaming keys while the sample pass runs and waits only before it
// reads tau; the finish pass waits for the scorer's lists.
//   1. topk_sample_kernel (this file): per query, score a sample of about
//      1/32 of its eligible entries (groups of 16 consecutive entries spread
//      evenly over them, on the tensor cores; 4-bit keys on the CUDA cores)
//      and set a threshold tau a few standard deviations below the sample's
//      estimate of the k-th largest key, so that about 2k keys reach it.
//   2. the scorer (indexer_tc.cu / indexer.cu / indexer_fp4.cu): every key
//      that reaches tau is appended, with its entry index, to the query's
//      candidate list of cand_cap slots; all of them are counted.
//   3. topk_finish_kernel (this file): if the count c satisfies
//      k <= c <= cand_cap, the k largest keys are all candidates (at least k
//      keys reach tau, and every key that reaches it was listed), so an exact
//      radix select over the candidates finishes the job.  Otherwise (tau was
//      too high or too low, which the sample makes rare for unstructured data)
//      the query's keys are recomputed here, exactly, in a few passes: a
//      12-bit histogram, refinements of the threshold bin, then a bitmap pass.
// Both branches give every key above the k-th largest, then the lowest-index
// keys equal to it, in ascending index order (bitmap compaction).
//
// Many-query mode (prefill, more than kFusedMaxQueries queries on one
// sequence) takes the same three steps with the per-query launches replaced:
// the tcgen05 scorer's sample pass scores a few whole key chunks per block of
// queries, topk_threshold_many_kernel derives tau per query (one warp each),
// and topk_finish_many_kernel selects among the candidates (one warp each),
// listing the queries whose count misses [k, cand_cap] for the recompute of
// topk_finish_kernel.
//
// Recomputed keys (sample and fallback) use plain fp32 arithmetic; they can
// differ from the scorer's in the last bits, which only moves near-ties.  The
// sample never affects the result, only how many candidates are kept.
#include <cooperative_groups.h>

#include "kernels.h"
#include "lowprec.cuh"
#include "score_mma.cuh"
#include "select.cuh"

namespace csa {

namespace {

constexpr int kSampleThreads = 256;            // sample pass: 8 warps per query
constexpr int kThreads = 512;                  // finish pass: 16 warps per query
constexpr int kSampleMin = 1024;               // sampled entries per query, at least
constexpr int kSampleMax = 16384;              // = kMaxSelectEntries / 32
constexpr int kHist = 4096;                    // first radix level of the fallback (12 bits)
constexpr int kCandSmem = 4096;                // fallback candidates held in shared memory
constexpr size_t kFinishSmem = 200 * 1024;     // dynamic shared memory of the finish kernel, at most
constexpr int kRankList = 512;                 // threshold-bin entries ranked directly

__device__ __forceinline__ int64_t eligible_of(const IndexerArgs& a, int64_t t) {
  const int64_t pos = a.q_pos ? __ldg(a.q_pos + t) : t;
  const int64_t n = pos / a.m;
  return n < a.max_entries ? n : a.max_entries;
}

// ---------------------------------------------------------------------------
// CUDA-core scoring of single entries (the sample and the fallback)
// ---------------------------------------------------------------------------
// The query's heads as fp32 in shared memory, [H_I][CI] (in 4-bit mode the
// dequantized E2M1 codes of the same block quantizer the 4-bit scorer uses),
// and its head weights [H_I].  Every thread of the block must call it.
template <int CI>
__device__ void load_query(const IndexerArgs& a, int64_t t, float* qs, float* ws) {
  if (!a.fp4) {
    const __nv_bfloat16* q = a.q_idx + t * a.H_I * CI;
    for (int i = threadIdx.x; i < a.H_I * CI; i += blockDim.x) qs[i] = __bfloat162float(q[i]);
  } else {
    for (int b = threadIdx.x; b < a.H_I * (CI / 32); b += blockDim.x) {
      const int h = b / (CI / 32), v = b - h * (CI / 32);
      uint32_t w4[4];
      const uint32_t sb = lowprec::quantize_block(a.q_idx + (t * a.H_I + h) * CI + 32 * v, w4);
      const float f = lowprec::e8m0_to_float(sb);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j)
          qs[h * CI + 32 * v + 8 * i + j] = lowprec::e2m1_to_float((w4[i] >> (4 * j)) & 15u) * f;
    }
  }
  for (int h = threadIdx.x; h < a.H_I; h += blockDim.x) ws[h] = __ldg(a.w + t * a.H_I + h);
}

// Score of the entry at physical row `row` (or of a zero key when row < 0,
// an entry the cache cannot address, which the scorer reports).  The key is
// read 64 dims at a time with every load of a batch issued before any is
// used; heads are taken 16 at a time, so that the accumulators stay in
// registers (the row is re-read from cache for each further group of 16
// heads or 64 dims).
template <int CI>
__device__ float entry_score(const IndexerArgs& a, const float* qs, const float* ws, int64_t row) {
  float s = 0.f;
  if (row < 0) return s;
  constexpr int CH = 64;   // dims per register batch
#pragma unroll 1
  for (int h0 = 0; h0 < a.H_I; h0 += 16) {
    float acc[16];
#pragma unroll
    for (int h = 0; h < 16; ++h) acc[h] = 0.f;
#pragma unroll 1
    for (int c0 = 0; c0 < CI; c0 += CH) {
      uint32_t raw[CH / 2];   // bf16 pairs, or code words (8 codes) in the first CH / 8
      float fsc[CH / 32];
      if (!a.fp4) {
        const uint4* p = reinterpret_cast<const uint4*>(a.keys.data + row * CI + c0);
#pragma unroll
        for (int i = 0; i < CH / 8; ++i) {
          const uint4 u = __ldg(p + i);
          raw[4 * i] = u.x;
          raw[4 * i + 1] = u.y;
          raw[4 * i + 2] = u.z;
          raw[4 * i + 3] = u.w;
        }
      } else {
        const uint4* p = reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(a.keys.data) +
                                                        row * (CI / 2) + c0 / 2);
#pragma unroll
        for (int i = 0; i < CH / 32; ++i) {
          const uint4 u = __ldg(p + i);
          raw[4 * i] = u.x;
          raw[4 * i + 1] = u.y;
          raw[4 * i + 2] = u.z;
          raw[4 * i + 3] = u.w;
        }
#pragma unroll
        for (int i = 0; i < CH / 32; ++i)
          fsc[i] = lowprec::e8m0_to_float(__ldg(a.k_scales + row * (CI / 32) + c0 / 32 + i));
      }
#pragma unroll
      for (int c = 0; c < CH / 8; ++c) {
        float k[8];
        if (!a.fp4) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 f = unpack_bf16(raw[4 * c + j]);
            k[2 * j] = f.x;
            k[2 * j + 1] = f.y;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) k[j] = lowprec::e2m1_to_float((raw[c] >> (4 * j)) & 15u) * fsc[c / 4];
        }
#pragma unroll
        for (int h = 0; h < 16; ++h) {
          if (h0 + h < a.H_I) {
            const float* qh = qs + (h0 + h) * CI + c0 + 8 * c;
            const float4 q0 = *reinterpret_cast<const float4*>(qh);
            const float4 q1 = *reinterpret_cast<const float4*>(qh + 4);
            float d = acc[h];
            d = fmaf(q0.x, k[0], d);
            d = fmaf(q0.y, k[1], d);
            d = fmaf(q0.z, k[2], d);
            d = fmaf(q0.w, k[3], d);
            d = fmaf(q1.x, k[4], d);
            d = fmaf(q1.y, k[5], d);
            d = fmaf(q1.z, k[6], d);
            d = fmaf(q1.w, k[7], d);
            acc[h] = d;
          }
        }
      }
    }
#pragma unroll
    for (int h = 0; h < 16; ++h)
      if (h0 + h < a.H_I) s = fmaf(ws[h0 + h], fmaxf(acc[h], 0.f), s);
  }
  return s;
}

// The fallback's key of entry j of sequence seq (kept out of line: the
// finish kernel calls it from several rarely taken passes).
template <int CI>
__device__ __noinline__ uint32_t recompute_key(const IndexerArgs& a, const float* qs,
                                               const float* ws, int32_t seq, int64_t j, int32_t t) {
  const int64_t row = cache_row(a.keys, seq, j, a.err, t);
  return score_key(entry_score<CI>(a, qs, ws, row));
}

// ---------------------------------------------------------------------------
// 1. sample and threshold
// ---------------------------------------------------------------------------
// tau from ns sampled keys in shared memory: the r-th largest of them with
// its low 10 bits cleared (two radix levels of 11 bits: bits 31-21, 20-10),
// r = the expected number of sampled keys at or above the k-th largest key
// plus six standard deviations and a margin; 0 when r reaches ns.
// With `built`, hist already holds the first level (bits 31-21 of every
// sampled key, counted while scoring).
template <int NT>
__device__ uint32_t sample_threshold(const uint32_t* skey, int ns, int64_t n, int top_k,
                                     int* hist, int* warp_sums, uint32_t* s_bin, int* s_above,
                                     int* s_ok, bool built = false) {
  const double mu = (double)ns * (double)top_k / (double)n;
  const int64_t r = (int64_t)ceil(mu + 6.0 * sqrt(mu) + 8.0);
  if (r >= ns) return 0u;
  uint32_t prefix = 0u;
  int need = (int)r;
#pragma unroll 1
  for (int level = 0; level < 2; ++level) {
    const int lo = level == 0 ? 21 : 10;
    if (level > 0 || !built) {
      for (int b = threadIdx.x; b < 2048; b += NT) hist[b] = 0;
      __syncthreads();
      for (int j = threadIdx.x; j < ns; j += NT) {
        const uint32_t key = skey[j];
        if (level == 0 || (key >> 21) == (prefix >> 21)) atomicAdd(&hist[(key >> lo) & 2047u], 1);
      }
      __syncthreads();
    }
    sel::find_bin<NT>(hist, 2048, need, warp_sums, s_bin, s_above, s_ok);
    prefix |= *s_bin << lo;
    need -= *s_above;
    __syncthreads();
  }
  return prefix;
}

// The same threshold for ns <= kWarpSample keys, by one warp without
// shared-memory histograms or block barriers: the keys go to registers (32
// per lane) and a bitwise radix select walks bits 31 .. 10 from the top, each
// step counting the keys of the current prefix group that have the bit set.
constexpr int kWarpSample = 1024;
__device__ uint32_t warp_sample_threshold(const uint32_t* skey, int ns, int64_t n, int top_k) {
  const double mu = (double)ns * (double)top_k / (double)n;
  const int64_t r = (int64_t)ceil(mu + 6.0 * sqrt(mu) + 8.0);
  if (r >= ns) return 0u;
  const int lane = threadIdx.x & 31;
  uint32_t kv[kWarpSample / 32];
#pragma unroll
  for (int i = 0; i < kWarpSample / 32; ++i) kv[i] = 32 * i + lane < ns ? skey[32 * i + lane] : 0u;
  uint32_t prefix = 0u;
  int need = (int)r;
#pragma unroll 1
  for (int bit = 31; bit >= 10; --bit) {
    const uint32_t want = (prefix >> bit) | 1u;
    int cnt = 0;
#pragma unroll
    for (int i = 0; i < kWarpSample / 32; ++i) cnt += (32 * i + lane < ns && (kv[i] >> bit) == want) ? 1 : 0;
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (cnt >= need) prefix |= 1u << bit;
    else need -= cnt;
  }
  return prefix;
}

// Sampled entries: ns = max(1024, n/32) (at most n, a multiple of 16), as
// ns / 16 groups of 16 consecutive entries, group i starting at i n / (ns/16).
__host__ __device__ __forceinline__ int sample_size(int64_t n) {
  int64_t ns = n / 32 > kSampleMin ? n / 32 : kSampleMin;
  if (ns > n) ns = n;
  if (ns > kSampleMax) ns = kSampleMax;
  return (int)(ns & ~int64_t(15));
}

// bf16 keys: C CTAs per query (a thread-block cluster when C > 1), each
// scoring its share of the groups of 16 entries with mma.sync (kU groups with
// their loads in flight at a time) into its own shared memory; with C > 1 the
// first CTA gathers the keys through distributed shared memory.  The first CTA
// sets tau: one warp's register select for samples of up to kWarpSample keys
// on one CTA, else the block-wide select.  C = 1 leaves most SMs to the scorer
// that overlaps this pass; large samples (long contexts) take C = 4.
// Dynamic shared memory: sample keys [kSampleMax] (each CTA fills the slots of
// its groups).
constexpr int kSampleCluster = 4;
template <int CI, int NT, int C>
__global__ void __launch_bounds__(kSampleThreads) topk_sample_kernel(IndexerArgs a, int top_k) {
  namespace cg = cooperative_groups;
  constexpr int kU = (CI == 128 && NT >= 4) ? 2 : (CI == 128 || NT >= 4) ? 4 : 8;
  extern __shared__ uint32_t skey[];
  __shared__ int hist[2048];
  __shared__ int warp_sums[32];
  __shared__ uint32_t s_bin;
  __shared__ int s_above, s_ok;

  pdl_trigger();   // the scorer may start streaming keys; it waits before it reads tau
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = C > 1 ? (int)cluster.block_rank() : 0;
  const int64_t tl = blockIdx.x / C;
  const int64_t t = a.t_begin + tl;
  if (threadIdx.x == 0 && rank == 0) a.cand_count[tl] = 0u;
  // the query's position, sequence and head fragments load together
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, q4 = lane & 3;
  const int64_t n = eligible_of(a, t);
  const int32_t seq = a.seq_id ? __ldg(a.seq_id + t) : 0;
  QueryFrags<CI, NT> Q;
  Q.load(a, t, g, q4);
  // few entries: every key is a candidate (cand_cap >= 2 top_k), nothing to
  // sample (the same for every CTA of the cluster: none waits at its barriers)
  if (n <= a.skip_le || 2 * n <= a.cand_cap) {
    if (threadIdx.x == 0 && rank == 0) const_cast<uint32_t*>(a.tau)[tl] = 0u;
    return;
  }
  const int ns = sample_size(n);
  const int ng = ns / 16;
  const int g_hi = (rank + 1) * ng / C;   // this CTA's groups: [rank ng / C, g_hi)
  for (int g0 = rank * ng / C + warp * kU; g0 < g_hi; g0 += (kSampleThreads / 32) * kU) {
    uint4 kr[kU][2][CI / 32];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int grp = g0 + u;
      const int64_t e0 = (int64_t)grp * n / ng;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t row = grp < g_hi ? cache_row(a.keys, seq, e0 + g + 8 * h, nullptr, 0) : -1;
#pragma unroll
        for (int v = 0; v < CI / 32; ++v)
          kr[u][h][v] = row >= 0 ? ld_stream_16(a.keys.data + row * CI + 32 * v + 8 * q4)
                                 : make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      float sg, s8;
      score_group<CI, NT>(kr[u], Q, sg, s8);
      const int grp = g0 + u;
      if (grp < g_hi && q4 < 2) skey[grp * 16 + g + 8 * q4] = score_key(q4 == 0 ? sg : s8);
    }
  }
  if (C > 1) {
    cluster.sync();   // every CTA's keys are in its shared memory
    if (rank == 0) {
      for (int r = 1; r < C; ++r) {
        const uint32_t* rk = cluster.map_shared_rank(skey, r);
        const int lo = (r * ng / C) * 16, hi = ((r + 1) * ng / C) * 16;
        for (int i = lo + (int)threadIdx.x; i < hi; i += kSampleThreads) skey[i] = rk[i];
      }
    }
    cluster.sync();   // the other CTAs' keys have been read before any of them exits
    if (rank != 0) return;
  } else {
    __syncthreads();
    if (ns <= kWarpSample) {   // the common case: one warp sets tau
      if (warp == 0) {
        const uint32_t tau = warp_sample_threshold(skey, ns, n, top_k);
        if (lane == 0) const_cast<uint32_t*>(a.tau)[tl] = tau;
      }
      return;
    }
  }
  const uint32_t tau = sample_threshold<kSampleThreads>(skey, ns, n, top_k, hist, warp_sums, &s_bin,
                                                        &s_above, &s_ok);
  if (threadIdx.x == 0) const_cast<uint32_t*>(a.tau)[tl] = tau;
}

// 4-bit keys: one thread per sampled entry on the CUDA cores (dequantized
// query in shared memory).  Dynamic shared memory: sample keys [kSampleMax],
// q [H_I * CI] fp32, w [64].
template <int CI>
__global__ void __launch_bounds__(kSampleThreads) topk_sample_fp4_kernel(IndexerArgs a, int top_k) {
  extern __shared__ uint32_t tsm[];
  uint32_t* skey = tsm;
  float* qs = reinterpret_cast<float*>(tsm + kSampleMax);
  float* ws = qs + a.H_I * CI;
  __shared__ int hist[2048];
  __shared__ int warp_sums[32];
  __shared__ uint32_t s_bin;
  __shared__ int s_above, s_ok;

  pdl_trigger();
  const int64_t tl = blockIdx.x;
  const int64_t t = a.t_begin + tl;
  if (threadIdx.x == 0) a.cand_count[tl] = 0u;
  const int64_t n = eligible_of(a, t);
  if (n <= a.skip_le || 2 * n <= a.cand_cap) {
    if (threadIdx.x == 0) const_cast<uint32_t*>(a.tau)[tl] = 0u;
    return;
  }
  const int ns = sample_size(n);
  const int ng = ns / 16;
  load_query<CI>(a, t, qs, ws);
  __syncthreads();
  const int32_t seq = a.seq_id ? __ldg(a.seq_id + t) : 0;
  for (int j = threadIdx.x; j < ns; j += kSampleThreads) {
    const int64_t e = (int64_t)(j >> 4) * n / ng + (j & 15);
    const int64_t row = cache_row(a.keys, seq, e, nullptr, 0);
    skey[j] = score_key(entry_score<CI>(a, qs, ws, row));
  }
  __syncthreads();
  if (ns <= kWarpSample) {
    if (threadIdx.x < 32) {
      const uint32_t tau = warp_sample_threshold(skey, ns, n, top_k);
      if (threadIdx.x == 0) const_cast<uint32_t*>(a.tau)[tl] = tau;
    }
    return;
  }
  const uint32_t tau =
      sample_threshold<kSampleThreads>(skey, ns, n, top_k, hist, warp_sums, &s_bin, &s_above, &s_ok);
  if (threadIdx.x == 0) const_cast<uint32_t*>(a.tau)[tl] = tau;
}

// ---------------------------------------------------------------------------
// 3. exact selection
// ---------------------------------------------------------------------------
struct FinishArgs {
  int top_k;
  int32_t* idx_out;
  int32_t* count_out;
  float* score_out;
  int stage_cap;                   // candidates that fit the shared-memory staging area
  const uint32_t* list = nullptr;  // with list: the queries list[0 .. *list_count) only,
  const uint32_t* list_count = nullptr;   // each CTA taking every gridDim.x-th
};

// A query with at most k eligible entries selects every one (ascending,
// padded with -1); when scores are asked for, the scorer listed all of them
// (tau = 0, no skipping).  Threads r, r + step, ... of the calling group.
__device__ __forceinline__ void finish_all_eligible(const IndexerArgs& a, const FinishArgs& f, int64_t t,
                                                    int64_t tl, int64_t n, int r, int step) {
  const int k = f.top_k;
  int32_t* idx = f.idx_out + t * k;
  float* sco = f.score_out ? f.score_out + t * k : nullptr;
  for (int64_t j = r; j < k; j += step) {
    idx[j] = j < n ? (int32_t)j : -1;
    if (sco && j >= n) sco[j] = -INFINITY;
  }
  if (sco) {
    const uint2* cand = a.cand + tl * a.cand_cap;
    const int64_t c_all = (int64_t)a.cand_count[tl];
    const int64_t c = c_all < a.cand_cap ? c_all : a.cand_cap;
    for (int64_t i = r; i < c; i += step) {
      const uint2 e = cand[i];
      if ((int64_t)e.y < n) sco[e.y] = key_score(e.x);
    }
  }
  if (r == 0) f.count_out[t] = (int32_t)n;
}

// Dynamic shared memory: sel [Wmax], tie [Wmax] (Wmax = ceil(max_entries/32)
// rounded up to a multiple of 4), a staging area of stage_cap (key, entry)
// pairs (the candidates, or the fallback's keys and ids [kCandSmem] each), q
// [H_I * CI] fp32, w [64].
template <int CI>
__global__ void __launch_bounds__(kThreads) topk_finish_kernel(IndexerArgs a, FinishArgs f) {
  extern __shared__ uint32_t fsm[];
  __shared__ int hist[kHist];
  __shared__ int warp_sums[32];
  __shared__ uint32_t s_bin;
  __shared__ int s_above, s_ok, s_overflow;
  __shared__ int s_wcnt[kThreads / 32];
  __shared__ uint32_t s_min[32], s_max[32];
  __shared__ int s_listn;

  pdl_wait();      // the scorer's candidate lists are complete
  pdl_trigger();
  auto finish_query = [&](const int64_t tl) {
    const int64_t t = a.t_begin + tl;
    const int64_t n = eligible_of(a, t);
    const int k = f.top_k;
    int32_t* idx = f.idx_out + t * k;
    float* sco = f.score_out ? f.score_out + t * k : nullptr;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint2* cand = a.cand + tl * a.cand_cap;
    const int64_t c_all = (int64_t)a.cand_count[tl];

    if (n <= k) {
      finish_all_eligible(a, f, t, tl, n, tid, kThreads);
      return;
    }

    const int W = (int)((n + 31) >> 5);
    const int Wmax = (int)((((a.max_entries + 31) >> 5) + 3) & ~int64_t(3));   // keeps q 16-byte aligned
    uint32_t* selb = fsm;
    uint32_t* tieb = fsm + Wmax;
    uint2* stage = reinterpret_cast<uint2*>(tieb + Wmax);
    uint32_t* cand_key = reinterpret_cast<uint32_t*>(stage);
    int32_t* cand_idx = reinterpret_cast<int32_t*>(cand_key + kCandSmem);
    float* qs = reinterpret_cast<float*>(stage + f.stage_cap);
    float* ws = qs + a.H_I * CI;
    for (int w = tid; w < W; w += kThreads) {
      selb[w] = 0u;
      tieb[w] = 0u;
    }
    bool consistent = true;
    int need;   // copies of the k-th largest key still to take, lowest index first

    if (c_all >= k && c_all <= a.cand_cap) {
      // ------------------------------------------------ select among candidates
      const int c = (int)c_all;
      // one pass over the list in global memory: staged in shared memory when
      // it fits (every later pass then stays on chip), and its key range
      const uint2* src = cand;
      uint32_t kmin = 0xffffffffu, kmax = 0u;
      if (c <= f.stage_cap) {
        // pairs of candidates as 16-byte vectors, four vectors of loads in
        // flight per thread before any is stored
        const uint4* g4 = reinterpret_cast<const uint4*>(cand);   // rows of cand_cap pairs: 16-byte aligned
        uint4* s4 = reinterpret_cast<uint4*>(stage);
        const int nv = (c + 1) >> 1;
        for (int i0 = tid; i0 < nv; i0 += 4 * kThreads) {
          uint4 v[4];
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (i0 + u * kThreads < nv) v[u] = __ldcs(g4 + i0 + u * kThreads);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i = i0 + u * kThreads;
            if (i < nv) {
              s4[i] = v[u];
              kmin = min(kmin, v[u].x);
              kmax = max(kmax, v[u].x);
              if (2 * i + 1 < c) {
                kmin = min(kmin, v[u].z);
                kmax = max(kmax, v[u].z);
              }
            }
          }
        }
        src = stage;
      } else {
        for (int i = tid; i < c; i += kThreads) {
          const uint32_t key = cand[i].x;
          kmin = min(kmin, key);
          kmax = max(kmax, key);
        }
      }
      for (int b = tid; b < kHist; b += kThreads) hist[b] = 0;
      if (tid == 0) s_listn = 0;
      kmin = __reduce_min_sync(0xffffffffu, kmin);
      kmax = __reduce_max_sync(0xffffffffu, kmax);
      if (lane == 0) {
        s_min[warp] = kmin;
        s_max[warp] = kmax;
      }
      __syncthreads();
      kmin = __reduce_min_sync(0xffffffffu, lane < kThreads / 32 ? s_min[lane] : 0xffffffffu);
      kmax = __reduce_max_sync(0xffffffffu, lane < kThreads / 32 ? s_max[lane] : 0u);
      // the candidates' common leading bits are fixed; the next 12 bits are a
      // digit (widened downwards to at least 512 bins, whose upper bits are then
      // fixed too)
      const int cpl = __clz(kmin ^ kmax);   // 32 when all candidates are equal
      uint32_t mask = cpl >= 32 ? 0xffffffffu : ~(0xffffffffu >> cpl);
      uint32_t prefix = kmin & mask;
      need = k;
      int shift = 32 - cpl;
      if (shift > 0) {
        const int lo = shift > 12 ? shift - 12 : 0;
        const int dig = shift - lo >= 9 ? shift - lo : 9;
        const uint32_t dmask = (1u << dig) - 1u;
        for (int i = tid; i < c; i += kThreads) atomicAdd(&hist[(src[i].x >> lo) & dmask], 1);
        __syncthreads();
        consistent &= sel::find_bin<kThreads>(hist, 1 << dig, need, warp_sums, &s_bin, &s_above, &s_ok);
        const uint32_t bsel = s_bin;
        const int in_bin = hist[bsel];
        need -= s_above;
        __syncthreads();   // the bins are read: hist becomes the threshold bin's list
        uint2* list = reinterpret_cast<uint2*>(hist);
        // keys above the threshold bin are selected; the bin's keys are listed
        // when few enough to rank directly
        const bool rank_list = in_bin <= kRankList;
        for (int i = tid; i < c; i += kThreads) {
          const uint2 e = src[i];
          if ((int64_t)e.y >= n) continue;   // never listed; kept out of the bitmaps
          const uint32_t dgt = (e.x >> lo) & dmask;
          if (dgt > bsel) {
            atomicOr(&selb[e.y >> 5], 1u << (e.y & 31));
          } else if (dgt == bsel && rank_list) {
            const int q = atomicAdd(&s_listn, 1);
            if (q < kRankList) list[q] = e;
          }
        }
        __syncthreads();
        if (rank_list) {
          // an entry of the bin is selected iff fewer than `need` entries of the
          // bin come before it in (key descending, index ascending) order: this
          // also settles ties at the k-th key by the lower index
          const int mb = s_listn < kRankList ? s_listn : kRankList;
          for (int q = tid; q < mb; q += kThreads) {
            const uint2 e = list[q];
            int before = 0;
            for (int j = 0; j < mb; ++j) {
              const uint2 o = list[j];
              before += (o.x > e.x) || (o.x == e.x && o.y < e.y);
            }
            if (before < need) atomicOr(&selb[e.y >> 5], 1u << (e.y & 31));
          }
          need = 0;
        } else {
          // a crowded bin: further 11-bit digits over the candidates, then the
          // k-th key's copies go to the lowest indices
          prefix |= bsel << lo;
          mask |= dmask << lo;
          shift = lo;
#pragma unroll 1
          while (shift > 0) {
            const int lo2 = shift > 11 ? shift - 11 : 0;
            const int dig2 = shift - lo2 >= 9 ? shift - lo2 : 9;
            const uint32_t dm2 = (1u << dig2) - 1u;
            for (int b = tid; b < (1 << dig2); b += kThreads) hist[b] = 0;
            __syncthreads();
            for (int i = tid; i < c; i += kThreads) {
              const uint32_t key = src[i].x;
              if ((key & mask) == prefix) atomicAdd(&hist[(key >> lo2) & dm2], 1);
            }
            __syncthreads();
            consistent &= sel::find_bin<kThreads>(hist, 1 << dig2, need, warp_sums, &s_bin, &s_above, &s_ok);
            prefix |= s_bin << lo2;
            mask |= dm2 << lo2;
            need -= s_above;
            shift = lo2;
            __syncthreads();
          }
          for (int i = tid; i < c; i += kThreads) {
            const uint2 e = src[i];
            if ((int64_t)e.y >= n) continue;
            if (e.x > prefix) atomicOr(&selb[e.y >> 5], 1u << (e.y & 31));
            else if (e.x == prefix) atomicOr(&tieb[e.y >> 5], 1u << (e.y & 31));
          }
        }
      } else {
        // every candidate has the same key: the lowest indices win
        for (int i = tid; i < c; i += kThreads) {
          const uint2 e = src[i];
          if ((int64_t)e.y < n) atomicOr(&tieb[e.y >> 5], 1u << (e.y & 31));
        }
      }
      __syncthreads();
    } else {
      // ------------------------------------------------ fallback: recompute
      load_query<CI>(a, t, qs, ws);
      __syncthreads();
      const int32_t seq = a.seq_id ? __ldg(a.seq_id + t) : 0;
      auto key_at = [&](int64_t j) -> uint32_t {
        return recompute_key<CI>(a, qs, ws, seq, j, (int32_t)t);
      };
      for (int b = tid; b < kHist; b += kThreads) hist[b] = 0;
      __syncthreads();
      for (int64_t j = tid; j < n; j += kThreads) atomicAdd(&hist[key_at(j) >> 20], 1);
      __syncthreads();
      consistent &= sel::find_bin<kThreads>(hist, kHist, k, warp_sums, &s_bin, &s_above, &s_ok);
      uint32_t prefix = s_bin << 20, mask = 0xfff00000u;
      need = k - s_above;
      int cnt = hist[s_bin];
      int shift = 20;
      __syncthreads();
      // refine the prefix by one 10-bit digit with a recompute pass
      auto refine = [&]() {
        shift -= 10;
        for (int b = tid; b < 1024; b += kThreads) hist[b] = 0;
        __syncthreads();
        for (int64_t j = tid; j < n; j += kThreads) {
          const uint32_t key = key_at(j);
          if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 1023u], 1);
        }
        __syncthreads();
        consistent &= sel::find_bin<kThreads>(hist, 1024, need, warp_sums, &s_bin, &s_above, &s_ok);
        prefix |= s_bin << shift;
        mask |= 1023u << shift;
        need -= s_above;
        cnt = hist[s_bin];
        __syncthreads();
      };
      while (cnt > kCandSmem && shift > 0) refine();
      constexpr int kWarpCap = kCandSmem / (kThreads / 32);
      // one pass per warp and word: keys above the prefix go to the bitmap;
      // keys equal to it are candidates in the warp's slice (or ties when the
      // prefix is complete); a slice overflow refines and repeats the pass
      for (;;) {
        if (tid == 0) s_overflow = 0;
        __syncthreads();
        int wcnt = 0;
        for (int w = warp; w < W; w += kThreads / 32) {
          const int64_t j = (int64_t)w * 32 + lane;
          const uint32_t key = j < n ? key_at(j) : 0u;
          const uint32_t mk = key & mask;
          const bool gt = j < n && mk > prefix;
          const bool eq = j < n && mk == prefix;
          const uint32_t bg = __ballot_sync(0xffffffffu, gt);
          const uint32_t be = __ballot_sync(0xffffffffu, eq);
          if (lane == 0) {
            selb[w] = bg;
            tieb[w] = shift == 0 ? be : 0u;
          }
          if (shift > 0 && be) {
            if (eq) {
              const int p = wcnt + __popc(be & ((1u << lane) - 1u));
              if (p < kWarpCap) {
                cand_key[warp * kWarpCap + p] = key;
                cand_idx[warp * kWarpCap + p] = (int32_t)j;
              }
            }
            wcnt += __popc(be);
          }
        }
        if (lane == 0) {
          s_wcnt[warp] = wcnt;
          if (wcnt > kWarpCap) s_overflow = 1;
        }
        __syncthreads();
        if (!s_overflow || shift == 0) break;
        refine();
      }
      if (shift > 0) {
        auto cand_ok = [&](int cc) { return (cc % kWarpCap) < s_wcnt[cc / kWarpCap]; };
        int nc = 0;
        for (int w = 0; w < kThreads / 32; ++w) nc += min(s_wcnt[w], kWarpCap);
        if (need >= nc) {
          for (int cc = tid; cc < kCandSmem; cc += kThreads)
            if (cand_ok(cc)) atomicOr(&selb[cand_idx[cc] >> 5], 1u << (cand_idx[cc] & 31));
          need = 0;
        } else {
          // radix select of the need-th largest candidate over the low bits
          uint32_t cp = prefix, cm = mask;
          while (shift > 0) {
            const int dig = shift >= 10 ? 10 : shift;
            shift -= dig;
            const uint32_t dm = (1u << dig) - 1u;
            for (int b = tid; b < 1024; b += kThreads) hist[b] = 0;
            __syncthreads();
            for (int cc = tid; cc < kCandSmem; cc += kThreads)
              if (cand_ok(cc) && (cand_key[cc] & cm) == cp) atomicAdd(&hist[(cand_key[cc] >> shift) & dm], 1);
            __syncthreads();
            consistent &= sel::find_bin<kThreads>(hist, 1024, need, warp_sums, &s_bin, &s_above, &s_ok);
            cp |= s_bin << shift;
            cm |= dm << shift;
            need -= s_above;
            __syncthreads();
          }
          for (int cc = tid; cc < kCandSmem; cc += kThreads) {
            if (!cand_ok(cc)) continue;
            const uint32_t key = cand_key[cc];
            const int j = cand_idx[cc];
            if (key > cp) atomicOr(&selb[j >> 5], 1u << (j & 31));
            else if (key == cp) atomicOr(&tieb[j >> 5], 1u << (j & 31));
          }
        }
      }
      __syncthreads();
      sel::take_lowest_ties<kThreads>(selb, tieb, W, need, warp_sums);
      sel::compact_ascending<kThreads>(selb, W, k, idx, warp_sums, [&](int o, int64_t j) {
        if (sco) sco[o] = key_score(key_at(j));
      });
      if (tid == 0) {
        f.count_out[t] = k;
        if (!consistent) report(a.err, kErrSelect, (int32_t)t, k);
      }
      return;
    }

    // ---------------------------------------------------- candidates: finish
    if (need > 0) sel::take_lowest_ties<kThreads>(selb, tieb, W, need, warp_sums);
    sel::compact_ascending<kThreads>(selb, W, k, idx, warp_sums, [](int, int64_t) {});
    if (sco) {
      // output position of a selected entry j = set bits of sel below j:
      // prefix counts per 1024 entries (32 words), then the words in between
      __syncthreads();
      int* gpre = hist;   // (W + 31) / 32 <= 512 groups
      const int G = (W + 31) >> 5;
      int cg = 0;
      if (tid < G)
        for (int w = tid * 32; w < min(W, tid * 32 + 32); ++w) cg += __popc(selb[w]);
      int tot;
      const int before = sel::block_exclusive_scan<kThreads>(cg, warp_sums, tot);
      if (tid < G) gpre[tid] = before;
      __syncthreads();
      const int c = (int)c_all;
      const uint2* src = c <= f.stage_cap ? stage : cand;
      for (int i = tid; i < c; i += kThreads) {
        const uint2 e = src[i];
        const uint32_t j = e.y;
        if ((int64_t)j >= n || !((selb[j >> 5] >> (j & 31)) & 1u)) continue;
        int pos = gpre[j >> 10];
        for (uint32_t w = (j >> 10) << 5; w < (j >> 5); ++w) pos += __popc(selb[w]);
        pos += __popc(selb[j >> 5] & ((1u << (j & 31)) - 1u));
        if (pos < k) sco[pos] = key_score(e.x);
      }
    }
    if (tid == 0) {
      f.count_out[t] = k;
      if (!consistent) report(a.err, kErrSelect, (int32_t)t, k);
    }
  };
  if (f.list == nullptr) {
    finish_query(blockIdx.x);
    return;
  }
  const int64_t nl = (int64_t)*f.list_count;
  for (int64_t i = blockIdx.x; i < nl; i += gridDim.x) {
    __syncthreads();   // the previous query's shared memory is no longer read
    finish_query((int64_t)f.list[i]);
  }
}

// ---------------------------------------------------------------------------
// Many-query mode (prefill): one warp per query in both passes below, so that
// tens of queries share an SM and no pass waits on a block-wide barrier.
// ---------------------------------------------------------------------------
// Warp-level helpers.  Histogram bins are owned from the top, nbins / 32 per
// lane (nbins a multiple of 32).
__device__ __forceinline__ int warp_exclusive_scan(int v, int& total) {
  const int lane = threadIdx.x & 31;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  total = __shfl_sync(0xffffffffu, x, 31);
  return x - v;
}

// Bin holding the need-th largest counted element: false (bin 0, above 0)
// when the histogram holds fewer than `need`.
__device__ __forceinline__ bool warp_find_bin(const int* hist, int nbins, int need, uint32_t& bin,
                                              int& above) {
  const int lane = threadIdx.x & 31, per = nbins >> 5;
  int c = 0;
  for (int r = 0; r < per; ++r) c += hist[nbins - 1 - (lane * per + r)];
  int tot;
  int before = warp_exclusive_scan(c, tot);
  uint32_t my_bin = 0u;
  int my_above = 0;
  const bool mine = before < need && before + c >= need;
  if (mine) {
    for (int r = 0; r < per; ++r) {
      const int b = nbins - 1 - (lane * per + r);
      const int h = hist[b];
      if (before + h >= need) {
        my_bin = (uint32_t)b;
        my_above = before;
        break;
      }
      before += h;
    }
  }
  const uint32_t who = __ballot_sync(0xffffffffu, mine);
  if (who == 0u) {
    bin = 0u;
    above = 0;
    return false;
  }
  const int src = __ffs(who) - 1;
  bin = __shfl_sync(0xffffffffu, my_bin, src);
  above = __shfl_sync(0xffffffffu, my_above, src);
  return true;
}

// The first `need` set bits of tie[0 .. W) (index order) join sel.
__device__ __forceinline__ void warp_take_lowest_ties(uint32_t* sel, const uint32_t* tie, int W, int need) {
  const int lane = threadIdx.x & 31;
  const int wpt = (W + 31) >> 5, w0 = lane * wpt, w1 = min(W, w0 + wpt);
  int c = 0;
  for (int w = w0; w < w1; ++w) c += __popc(tie[w]);
  int tot;
  int before = warp_exclusive_scan(c, tot);
  for (int w = w0; w < w1; ++w) {
    uint32_t x = tie[w];
    const int pc = __popc(x);
    int take = need - before;
    take = take < 0 ? 0 : (take > pc ? pc : take);
    uint32_t kept = 0u;
    for (int i = 0; i < take; ++i) {
      const uint32_t low = x & (0u - x);
      kept |= low;
      x ^= low;
    }
    sel[w] |= kept;
    before += pc;
  }
  __syncwarp();
}

// Threshold pass: tau of each query from the keys the scorer's sample pass
// left in psample (the few-query sample pass's rank rule, the same 10 low
// bits cleared); also zeroes the candidate counts, the fallback list and the
// work counter of the scoring pass that follows.
constexpr int kTWarps = 4;
__global__ void __launch_bounds__(kTWarps * 32) topk_threshold_many_kernel(IndexerArgs a, int top_k,
                                                                        int64_t t_count, int qb) {
  pdl_wait();      // the sample pass's keys are complete (and it no longer uses the work counter)
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    *a.fb_count = 0u;
    *a.work = 0u;
  }
  const int64_t tl = (int64_t)blockIdx.x * kTWarps + warp;
  if (tl >= t_count) return;
  const int64_t t = a.t_begin + tl;
  if (lane == 0) a.cand_count[tl] = 0u;
  const int64_t n = eligible_of(a, t);
  uint32_t tau = 0u;
  if (n > a.skip_le && 2 * n > a.cand_cap) {
    // the sampled chunks of the query's block of qb queries, by the scorer's rule
    const int64_t QB = qb;
    const int64_t b0 = tl / QB * QB, b1 = b0 + QB < t_count ? b0 + QB : t_count;
    int64_t nmin = INT64_MAX, nmax = 0;
    for (int64_t u = b0 + lane; u < b1; u += 32) {
      const int64_t nu = eligible_of(a, a.t_begin + u);
      nmin = nu < nmin ? nu : nmin;
      nmax = nu > nmax ? nu : nmax;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const int64_t x = __shfl_xor_sync(0xffffffffu, nmin, o), y = __shfl_xor_sync(0xffffffffu, nmax, o);
      nmin = x < nmin ? x : nmin;
      nmax = y > nmax ? y : nmax;
    }
    const int ns = 256 * psample_chunks(nmin, nmax, a.cand_cap, a.skip_le);
    const double mu = (double)ns * (double)top_k / (double)n;
    const int64_t r = (int64_t)ceil(mu + 6.0 * sqrt(mu) + 8.0);
    if (ns > 0 && r < ns) {
      // the r-th largest sampled key with its low 10 bits cleared, by a
      // bitwise radix select over the keys held in registers (32 per lane):
      // bit by bit from the top, the count of keys in the current prefix
      // group with that bit set decides the branch
      uint32_t kv[kPSampleKeys / 32];
      const uint32_t* sk = a.psample + tl * kPSampleKeys;
      const int nv = ns >> 5;   // ns is a multiple of 256: whole rows of 32
#pragma unroll
      for (int i = 0; i < kPSampleKeys / 32; ++i) kv[i] = i < nv ? __ldcs(sk + 32 * i + lane) : 0u;
      uint32_t prefix = 0u;
      int need = (int)r;
#pragma unroll 1
      for (int bit = 31; bit >= 10; --bit) {
        const uint32_t want = (prefix >> bit) | 1u;
        int cnt = 0;
#pragma unroll
        for (int i = 0; i < kPSampleKeys / 32; ++i) cnt += (i < nv && (kv[i] >> bit) == want) ? 1 : 0;
        cnt = __reduce_add_sync(0xffffffffu, cnt);
        if (cnt >= need) prefix |= 1u << bit;
        else need -= cnt;
      }
      tau = prefix;
    }
  }
  if (lane == 0) const_cast<uint32_t*>(a.tau)[tl] = tau;
}

// Finish pass: the exact top-k among a query's candidates by one warp, when
// top_k <= count <= cand_cap; other queries are appended to the fallback
// list for topk_finish_kernel's recompute.  Shared memory per warp: hist
// [1024] int, sel / tie bitmaps [Wmax] each, the threshold bin's list
// [kWList] (key, entry) pairs.
constexpr int kFWarps = 8;
constexpr int kWList = 128;
constexpr int kFBatch = 8;   // candidates per lane with their loads in flight together
__host__ __device__ inline int finish_many_words(int64_t max_entries) {
  return (int)((((max_entries + 31) >> 5) + 1) & ~int64_t(1));   // keeps the list 8-byte aligned
}
__global__ void __launch_bounds__(kFWarps * 32) topk_finish_many_kernel(IndexerArgs a, FinishArgs f,
                                                                     int64_t t_count) {
  extern __shared__ __align__(16) uint32_t msm[];
  pdl_wait();      // the scorer's candidate lists are complete
  pdl_trigger();   // the recompute launch may start; it waits for this one
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t tl = (int64_t)blockIdx.x * kFWarps + warp;
  if (tl >= t_count) return;   // no block-wide barrier below
  const int Wmax = finish_many_words(a.max_entries);
  uint32_t* my = msm + (size_t)warp * (1024 + 2 * Wmax + 2 * kWList);
  int* hist = reinterpret_cast<int*>(my);
  uint32_t* selb = my + 1024;
  uint32_t* tieb = selb + Wmax;
  uint2* list = reinterpret_cast<uint2*>(tieb + Wmax);

  const int64_t t = a.t_begin + tl;
  const int64_t n = eligible_of(a, t);
  const int k = f.top_k;
  int32_t* idx = f.idx_out + t * k;
  float* sco = f.score_out ? f.score_out + t * k : nullptr;
  const uint2* cand = a.cand + tl * a.cand_cap;
  const int64_t c_all = (int64_t)a.cand_count[tl];
  if (n <= k) {
    finish_all_eligible(a, f, t, tl, n, lane, 32);
    return;
  }
  if (c_all < k || c_all > a.cand_cap) {
    if (lane == 0) a.fb_list[atomicAdd(a.fb_count, 1u)] = (uint32_t)tl;
    return;
  }
  const int c = (int)c_all;
  const int W = (int)((n + 31) >> 5);
  for (int w = lane; w < W; w += 32) {
    selb[w] = 0u;
    tieb[w] = 0u;
  }
  // every pass walks the list kFBatch candidates per lane at a time, with all
  // of their loads issued before any is used; fn(e, in_range) is called by
  // every lane for each slot of the batch (warp-collective calls allowed)
  auto for_each_cand = [&](auto&& fn) {
    for (int i0 = 0; i0 < c; i0 += 32 * kFBatch) {
      uint2 e[kFBatch];
#pragma unroll
      for (int u = 0; u < kFBatch; ++u) {
        const int i = i0 + 32 * u + lane;
        e[u] = i < c ? cand[i] : make_uint2(0u, 0xffffffffu);
      }
#pragma unroll
      for (int u = 0; u < kFBatch; ++u) fn(e[u], i0 + 32 * u + lane < c);
    }
  };
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  for_each_cand([&](const uint2 e, bool in) {
    if (in) {
      kmin = min(kmin, e.x);
      kmax = max(kmax, e.x);
    }
  });
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  __syncwarp();
  const int cpl = __clz(kmin ^ kmax);   // 32 when all candidates are equal
  uint32_t mask = cpl >= 32 ? 0xffffffffu : ~(0xffffffffu >> cpl);
  uint32_t prefix = kmin & mask;
  int need = k;
  int shift = 32 - cpl;
  bool consistent = true;
  // digits of at most 10 bits below the common prefix until the threshold
  // bin is small enough to rank directly, or the key is complete
  while (shift > 0) {
    const int dig = shift < 10 ? shift : 10;
    const int lo = shift - dig;
    const uint32_t dm = (1u << dig) - 1u;
    const int nb = dig < 5 ? 32 : (1 << dig);
    for (int b = lane; b < nb; b += 32) hist[b] = 0;
    __syncwarp();
    for_each_cand([&](const uint2 e, bool in) {
      if (in && (e.x & mask) == prefix) atomicAdd(&hist[(e.x >> lo) & dm], 1);
    });
    __syncwarp();
    uint32_t bin;
    int above;
    consistent &= warp_find_bin(hist, nb, need, bin, above);
    const int in_bin = hist[bin];
    prefix |= bin << lo;
    mask |= dm << lo;
    need -= above;
    shift = lo;
    __syncwarp();
    if (in_bin <= kWList) break;
  }
  // keys above the threshold bin are selected; its keys are ties (complete
  // key) or listed for ranking
  int listn = 0;
  for_each_cand([&](const uint2 e, bool in) {
    const bool valid = in && (int64_t)e.y < n;
    const uint32_t mk = e.x & mask;
    if (valid && mk > prefix) atomicOr(&selb[e.y >> 5], 1u << (e.y & 31));
    const bool eq = valid && mk == prefix;
    if (shift == 0) {
      if (eq) atomicOr(&tieb[e.y >> 5], 1u << (e.y & 31));
    } else {
      const uint32_t be = __ballot_sync(0xffffffffu, eq);
      const int pos = listn + __popc(be & ((1u << lane) - 1u));
      if (eq && pos < kWList) list[pos] = e;
      listn += __popc(be);
    }
  });
  __syncwarp();
  if (shift > 0) {
    // an entry of the bin is selected iff fewer than `need` entries of the bin
    // precede it in (key descending, index ascending) order
    const int mb = listn < kWList ? listn : kWList;
    consistent &= listn <= kWList;
    for (int q = lane; q < mb; q += 32) {
      const uint2 e = list[q];
      int before = 0;
      for (int j = 0; j < mb; ++j) {
        const uint2 o = list[j];
        before += (o.x > e.x) || (o.x == e.x && o.y < e.y);
      }
      if (before < need) atomicOr(&selb[e.y >> 5], 1u << (e.y & 31));
    }
    need = 0;
  }
  __syncwarp();
  if (need > 0) warp_take_lowest_ties(selb, tieb, W, need);
  // ascending compaction: lane-owned runs of words, then (for the scores)
  // each word's output offset, kept in the tie bitmap's place
  const int wpt = (W + 31) >> 5, w0 = lane * wpt, w1 = min(W, w0 + wpt);
  int cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(selb[w]);
  int tot;
  int o = warp_exclusive_scan(cnt, tot);
  for (int w = w0; w < w1; ++w) {
    uint32_t x = selb[w];
    tieb[w] = (uint32_t)o;
    while (x) {
      const int b = __ffs(x) - 1;
      x &= x - 1;
      if (o < k) idx[o] = w * 32 + b;
      ++o;
    }
  }
  __syncwarp();
  if (sco) {
    for_each_cand([&](const uint2 e, bool in) {
      const uint32_t j = e.y;
      if (!in || (int64_t)j >= n || !((selb[j >> 5] >> (j & 31)) & 1u)) return;
      const uint32_t pos = tieb[j >> 5] + (uint32_t)__popc(selb[j >> 5] & ((1u << (j & 31)) - 1u));
      if (pos < (uint32_t)k) sco[pos] = key_score(e.x);
    });
  }
  if (lane == 0) {
    f.count_out[t] = k;
    if (!consistent || tot != k) report(a.err, kErrSelect, (int32_t)t, k);
  }
}

// The same selection for entry lists of at most kSmallList entries (every
// query's candidates then fit in registers: 32 per lane): one load of the
// list, then a bitwise radix select over the keys in registers, from the
// highest bit on which the keys differ, bit by bit: it stops as soon as the
// keys at or above the current prefix are exactly k (then no tie is left),
// else it ends with the exact k-th largest key T and how many keys equal to T
// are taken (lowest entries first).  Selected keys and ties go to the
// bitmaps, then the same ascending compaction.  No shared-memory histograms
// and no second pass over the list in memory.
constexpr int kSWarps = 4;         // queries (warps) per CTA
constexpr int kSmallList = 1024;   // longest entry list of this form
__global__ void __launch_bounds__(kSWarps * 32) topk_finish_small_kernel(IndexerArgs a, FinishArgs f,
                                                                       int64_t t_count) {
  __shared__ uint32_t sbits[kSWarps][2][kSmallList / 32];
  pdl_wait();      // the scorer's candidate lists are complete
  pdl_trigger();   // the recompute launch may start; it waits for this one
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t tl = (int64_t)blockIdx.x * kSWarps + warp;
  if (tl >= t_count) return;   // no block-wide barrier below
  const int64_t t = a.t_begin + tl;
  const int64_t n = eligible_of(a, t);
  const int k = f.top_k;
  int32_t* idx = f.idx_out + t * k;
  float* sco = f.score_out ? f.score_out + t * k : nullptr;
  const uint2* cand = a.cand + tl * a.cand_cap;
  const int64_t c_all = (int64_t)a.cand_count[tl];
  if (n <= k) {
    finish_all_eligible(a, f, t, tl, n, lane, 32);
    return;
  }
  if (c_all < k || c_all > a.cand_cap || c_all > kSmallList || n > kSmallList) {
    if (lane == 0) a.fb_list[atomicAdd(a.fb_count, 1u)] = (uint32_t)tl;
    return;
  }
  const int c = (int)c_all;
  const int W = (int)((n + 31) >> 5);
  uint32_t* selb = sbits[warp][0];
  uint32_t* tieb = sbits[warp][1];
  for (int w = lane; w < W; w += 32) {
    selb[w] = 0u;
    tieb[w] = 0u;
  }
  // candidate 32 j + lane in e[j]; a slot past the list, or an entry past
  // the eligible range, holds entry 0xffffffff (never valid)
  uint2 e[kSmallList / 32];
  uint32_t vm = 0u;   // bit j: e[j] is a candidate of an eligible entry
  uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
  for (int j = 0; j < kSmallList / 32; ++j) {
    const int i = 32 * j + lane;
    e[j] = i < c ? cand[i] : make_uint2(0u, 0xffffffffu);
    if (i < c && (int64_t)e[j].y < n) {
      vm |= 1u << j;
      kmin = min(kmin, e[j].x);
      kmax = max(kmax, e[j].x);
    }
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  // every eligible key shares the bits above hb; the loop walks bit hb down
  int need = k;
  uint32_t prefix = kmin;
  int stop = 0;          // lowest bit examined
  bool early = false;    // the keys whose bits stop.. match the prefix or more are exactly k
  if (kmin != kmax) {
    const int hb = 31 - __clz(kmin ^ kmax);
    prefix = hb == 31 ? 0u : kmin & (0xffffffffu << (hb + 1));
#pragma unroll 1
    for (int bit = hb; bit >= 0; --bit) {
      const uint32_t want = (prefix >> bit) | 1u;
      int cnt = 0;
#pragma unroll
      for (int j = 0; j < kSmallList / 32; ++j) cnt += ((vm >> j) & 1u) && (e[j].x >> bit) == want ? 1 : 0;
      cnt = __reduce_add_sync(0xffffffffu, cnt);
      stop = bit;
      if (cnt >= need) {
        prefix |= 1u << bit;
        if (cnt == need) {
          early = true;
          break;
        }
      } else {
        need -= cnt;
      }
    }
  }
  __syncwarp();
  // early: keys with (key >> stop) >= (prefix >> stop) are the k selected.
  // Else T = prefix: keys above it are selected, and `need` of the keys
  // equal to it (1 <= need <= their number), the lowest entries.
  const uint32_t thr = prefix >> stop;
  int ties = 0;
#pragma unroll
  for (int j = 0; j < kSmallList / 32; ++j) {
    if (!((vm >> j) & 1u)) continue;
    const uint32_t y = e[j].y, hi = e[j].x >> stop;
    if (hi > thr || (early && hi == thr)) atomicOr(&selb[y >> 5], 1u << (y & 31));
    else if (hi == thr) {
      atomicOr(&tieb[y >> 5], 1u << (y & 31));
      ++ties;
    }
  }
  ties = __reduce_add_sync(0xffffffffu, ties);
  bool consistent = early || (need >= 1 && need <= ties);
  if (early) need = 0;
  __syncwarp();
  if (need > 0) warp_take_lowest_ties(selb, tieb, W, need);
  // ascending compaction (n <= kSmallList: one bitmap word per lane), then
  // each word's output offset kept in the tie bitmap's place for the scores
  const uint32_t x0 = lane < W ? selb[lane] : 0u;
  int tot;
  const int o0 = warp_exclusive_scan(__popc(x0), tot);
  if (lane < W) tieb[lane] = (uint32_t)o0;
  {
    uint32_t x = x0;
    int o = o0;
    while (x) {
      const int b = __ffs(x) - 1;
      x &= x - 1;
      if (o < k) idx[o] = lane * 32 + b;
      ++o;
    }
  }
  __syncwarp();
  if (sco) {
#pragma unroll
    for (int j = 0; j < kSmallList / 32; ++j) {
      const uint32_t y = e[j].y;
      if (!((vm >> j) & 1u) || !((selb[y >> 5] >> (y & 31)) & 1u)) continue;
      const uint32_t pos = tieb[y >> 5] + (uint32_t)__popc(selb[y >> 5] & ((1u << (y & 31)) - 1u));
      if (pos < (uint32_t)k) sco[pos] = key_score(e[j].x);
    }
  }
  if (lane == 0) {
    f.count_out[t] = k;
    if (!consistent || tot != k) report(a.err, kErrSelect, (int32_t)t, k);
  }
}

template <int CI>
cudaError_t launch_finish(const Launch& L, const IndexerArgs& a, int top_k, int32_t* idx_out,
                          int32_t* count_out, float* score_out, int64_t t_count,
                          const uint32_t* list = nullptr, const uint32_t* list_count = nullptr) {
  const size_t qbytes = (size_t)a.H_I * CI * sizeof(float) + 64 * sizeof(float);
  const size_t wmax = (size_t)((((a.max_entries + 31) >> 5) + 3) & ~int64_t(3));
  // staging area: the whole candidate list when it fits next to the bitmaps
  // and the query (at least the fallback's 2 x kCandSmem words)
  const size_t fixed = 2 * wmax * sizeof(uint32_t) + qbytes;
  size_t stage = kFinishSmem > fixed ? (kFinishSmem - fixed) / 8 : 0;
  if (stage > (size_t)a.cand_cap) stage = (size_t)a.cand_cap;
  if (stage < (size_t)kCandSmem) stage = kCandSmem;
  stage &= ~size_t(1);
  const size_t bytes = fixed + stage * 8;
  cudaFuncSetAttribute(topk_finish_kernel<CI>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  prefer_max_shared(topk_finish_kernel<CI>);
  FinishArgs f{top_k, idx_out, count_out, score_out, (int)stage, list, list_count};
  return launch_kernel(topk_finish_kernel<CI>, dim3((unsigned)t_count), dim3(kThreads), bytes,
                       L.stream, list == nullptr, a, f);
}

// A sample kernel as clusters of kSampleCluster CTAs per query.
template <class K>
void launch_sample_cluster(K kernel, int64_t t_count, size_t smem, cudaStream_t stream, const IndexerArgs& a,
                           int top_k) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(t_count * kSampleCluster));
  cfg.blockDim = dim3(kSampleThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kSampleCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, kernel, a, top_k);
}

template <int CI>
void launch_sample(const Launch& L, const IndexerArgs& a, int top_k, int64_t t_count) {
  if (a.fp4) {
    const size_t bytes =
        kSampleMax * sizeof(uint32_t) + (size_t)a.H_I * CI * sizeof(float) + 64 * sizeof(float);
    prefer_max_shared(topk_sample_fp4_kernel<CI>);
    cudaFuncSetAttribute(topk_sample_fp4_kernel<CI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)bytes);
    topk_sample_fp4_kernel<CI><<<(unsigned)t_count, kSampleThreads, bytes, L.stream>>>(a, top_k);
    return;
  }
  const int nt = (a.H_I + 7) / 8;
  constexpr size_t kBytes = kSampleMax * sizeof(uint32_t);
  // one CTA per query while the largest sample fits one warp's select, else
  // clusters of kSampleCluster CTAs
  const bool clustered = sample_size(a.max_entries) > kWarpSample;
#define CSA_SAMPLE_CASE(NT_)                                                                   \
  if (nt <= NT_) {                                                                             \
    if (!clustered) {                                                                          \
      prefer_max_shared(topk_sample_kernel<CI, NT_, 1>);                                     \
      cudaFuncSetAttribute(topk_sample_kernel<CI, NT_, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                           (int)kBytes);                                                       \
      topk_sample_kernel<CI, NT_, 1><<<(unsigned)t_count, kSampleThreads, kBytes, L.stream>>>(a, top_k); \
    } else {                                                                                   \
      prefer_max_shared(topk_sample_kernel<CI, NT_, kSampleCluster>);                        \
      cudaFuncSetAttribute(topk_sample_kernel<CI, NT_, kSampleCluster>,                      \
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kBytes);          \
      launch_sample_cluster(topk_sample_kernel<CI, NT_, kSampleCluster>, t_count, kBytes, L.stream, a, top_k); \
    }                                                                                          \
    return;                                                                                    \
  }
  CSA_SAMPLE_CASE(1)
  CSA_SAMPLE_CASE(2)
  CSA_SAMPLE_CASE(4)
  CSA_SAMPLE_CASE(8)
#undef CSA_SAMPLE_CASE
}

}  // namespace

cudaError_t launch_topk_sample(const Launch& L, const IndexerArgs& a, int top_k, int64_t t_count) {
  if (t_count == 0) return cudaSuccess;
  L.begin(kKernelTopkSample);
  if (a.c_I == 64) launch_sample<64>(L, a, top_k, t_count);
  else launch_sample<128>(L, a, top_k, t_count);
  return L.end(kKernelTopkSample);
}

cudaError_t launch_topk_finish(const Launch& L, const IndexerArgs& a, int top_k, int32_t* idx_out,
                               int32_t* count_out, float* score_out, int64_t t_count) {
  if (t_count == 0) return cudaSuccess;
  L.begin(kKernelTopkSelect);
  if (a.c_I == 64) launch_finish<64>(L, a, top_k, idx_out, count_out, score_out, t_count);
  else launch_finish<128>(L, a, top_k, idx_out, count_out, score_out, t_count);
  return L.end(kKernelTopkSelect);
}

bool topk_many_supported(const IndexerArgs& a) {
  const size_t per_warp = (1024 + 2 * (size_t)finish_many_words(a.max_entries) + 2 * kWList) * 4;
  return a.fb_list != nullptr && a.fb_count != nullptr && per_warp * kFWarps <= 200 * 1024;
}

cudaError_t launch_topk_threshold_many(const Launch& L, const IndexerArgs& a, int top_k, int64_t t_count,
                                      int qb) {
  if (t_count == 0) return cudaSuccess;
  L.begin(kKernelTopkSample);
  prefer_max_shared(topk_threshold_many_kernel);
  const unsigned grid = (unsigned)((t_count + kTWarps - 1) / kTWarps);
  const cudaError_t e = launch_kernel(topk_threshold_many_kernel, dim3(grid), dim3(kTWarps * 32), 0, L.stream,
                                      true, a, top_k, t_count, qb);
  if (e != cudaSuccess) return e;
  return L.end(kKernelTopkSample);
}

cudaError_t launch_topk_finish_many(const Launch& L, const IndexerArgs& a, int top_k, int32_t* idx_out,
                                    int32_t* count_out, float* score_out, int64_t t_count) {
  if (t_count == 0) return cudaSuccess;
  L.begin(kKernelTopkSelect);
  const size_t bytes = (1024 + 2 * (size_t)finish_many_words(a.max_entries) + 2 * kWList) * 4 * kFWarps;
  cudaFuncSetAttribute(topk_finish_many_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  prefer_max_shared(topk_finish_many_kernel);
  FinishArgs f{top_k, idx_out, count_out, score_out, 0};
  if (a.max_entries <= kSmallList) {   // every list fits in registers
    const unsigned grid = (unsigned)((t_count + kSWarps - 1) / kSWarps);
    const cudaError_t e = launch_kernel(topk_finish_small_kernel, dim3(grid), dim3(kSWarps * 32), 0, L.stream,
                                        true, a, f, t_count);
    if (e != cudaSuccess) return e;
  } else {
    const unsigned grid = (unsigned)((t_count + kFWarps - 1) / kFWarps);
    const cudaError_t e = launch_kernel(topk_finish_many_kernel, dim3(grid), dim3(kFWarps * 32), bytes,
                                        L.stream, true, a, f, t_count);
    if (e != cudaSuccess) return e;
  }
  // the queries whose candidate count missed [top_k, cand_cap]: exact recompute
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t g2 = t_count < sms ? t_count : sms;
  if (a.c_I == 64) launch_finish<64>(L, a, top_k, idx_out, count_out, score_out, g2, a.fb_list, a.fb_count);
  else launch_finish<128>(L, a, top_k, idx_out, count_out, score_out, g2, a.fb_list, a.fb_count);
  return L.end(kKernelTopkSelect);
}

}  // namespace csa
