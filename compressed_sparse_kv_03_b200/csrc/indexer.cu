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
// permutation, which leaves every dot product unchanged.  Scores leave as
// order-preserving 32-bit keys; in the few-query (decode) mode each item also
// adds its keys to a 4096-bin histogram of the top 12 key bits.
//
// Selection is exact.  Decode mode (one CTA per query): the histogram gives
// the bin of the k-th largest key; if that bin is crowded, further 10-bit
// digits are refined with passes over the keys; one ballot pass then marks
// every key above the bin in a bitmap and collects the bin's keys as
// candidates; the candidates are resolved in shared memory; ties at the k-th
// key go to the lowest indices; a popcount scan of the bitmap writes the
// selected indices in ascending order.  Many-query (prefill) mode runs a
// three-digit radix select per query over its keys held in shared memory.
#include "kernels.h"

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
#ifndef CSA_SCORE_HIST_AGG
#define CSA_SCORE_HIST_AGG 0
#endif
constexpr int kScoreWarps = 8;
constexpr int kScoreThreads = kScoreWarps * 32;
constexpr int kUnroll = CSA_SCORE_UNROLL;   // 16-key groups in flight per warp

template <int CI, int NT>
struct QueryFrags {
  uint32_t bq[NT][CI / 16][2];
  float wv[NT][2];
  __device__ __forceinline__ void load(const IndexerArgs& a, int64_t t, int g, int q4) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int head = nt * 8 + g;
#pragma unroll
      for (int v = 0; v < CI / 32; ++v) {
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
  }
};

// Scores of rows g (sg) and g+8 (s8) of a 16-key group whose lanes hold
// r[h][v] = dims [32v + 8q, 32v + 8q + 8) of row g + 8h; summed over the quad.
template <int CI, int NT>
__device__ __forceinline__ void score_group(const uint4 (&r)[2][CI / 32],
                                            const QueryFrags<CI, NT>& Q, float& sg, float& s8) {
  sg = 0.f;
  s8 = 0.f;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int v = 0; v < CI / 32; ++v) {
      const uint32_t lo[4] = {r[0][v].x, r[1][v].x, r[0][v].y, r[1][v].y};
      mma_bf16_16816(d, lo, Q.bq[nt][2 * v][0], Q.bq[nt][2 * v][1]);
      const uint32_t hi[4] = {r[0][v].z, r[1][v].z, r[0][v].w, r[1][v].w};
      mma_bf16_16816(d, hi, Q.bq[nt][2 * v + 1][0], Q.bq[nt][2 * v + 1][1]);
    }
    sg = fmaf(Q.wv[nt][0], fmaxf(d[0], 0.f), sg);
    sg = fmaf(Q.wv[nt][1], fmaxf(d[1], 0.f), sg);
    s8 = fmaf(Q.wv[nt][0], fmaxf(d[2], 0.f), s8);
    s8 = fmaf(Q.wv[nt][1], fmaxf(d[3], 0.f), s8);
  }
  sg += __shfl_xor_sync(0xffffffffu, sg, 1);
  s8 += __shfl_xor_sync(0xffffffffu, s8, 1);
  sg += __shfl_xor_sync(0xffffffffu, sg, 2);
  s8 += __shfl_xor_sync(0xffffffffu, s8, 2);
}

// One CTA scores a chunk of `chunk` keys of one query (the grid is sized by
// the host to one resident wave).  Each warp walks 16-key groups with
// kUnroll groups of loads in flight; keys leave as order-preserving 32-bit
// keys, and in decode mode a shared histogram of their top 12 bits is added
// to the query's global histogram at the end.
template <int CI, int NT, bool HIST>
__global__ void __launch_bounds__(kScoreThreads, (CI == 64 && NT == 1) ? CSA_SCORE_MINBLOCKS : 1)
indexer_score_kernel(IndexerArgs a, int64_t chunk) {
  __shared__ uint32_t sh_hist[HIST ? kHistBins : 1];
  const int64_t tl = blockIdx.x;
  const int64_t t = a.t_begin + tl;
  const int64_t pos = a.q_pos ? __ldg(a.q_pos + t) : t;
  int64_t n_elig = pos / a.m;
  if (n_elig > a.max_entries) {
    if (blockIdx.y == 0 && threadIdx.x == 0) report(a.err, kErrEligible, (int32_t)t, n_elig);
    n_elig = a.max_entries;
  }
  const int64_t s_begin = (int64_t)blockIdx.y * chunk;
  if (s_begin >= n_elig) return;
  const int64_t s_end = min(s_begin + chunk, n_elig);
  const int32_t seq = a.seq_id ? __ldg(a.seq_id + t) : 0;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, q4 = lane & 3;
  if (HIST) {
    for (int b = threadIdx.x; b < kHistBins; b += kScoreThreads) sh_hist[b] = 0;
    __syncthreads();
  }
  QueryFrags<CI, NT> Q;
  Q.load(a, t, g, q4);
  uint32_t* out = a.keys_out + tl * a.key_stride;

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
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      float sg, s8;
      score_group<CI, NT>(kr[u], Q, sg, s8);
      const int64_t s = s0 + u * 16 + g + (q4 == 1 ? 8 : 0);
      const bool valid = q4 < 2 && s < s_end;
      const uint32_t key = score_key(q4 == 0 ? sg : s8);
      if (valid) out[s] = key;
      if (HIST) {
        if (CSA_SCORE_HIST_AGG) {   // one shared atomic per distinct bin of the warp
          const uint32_t bin = valid ? key >> 20 : 0xffffffffu;
          const uint32_t same = __match_any_sync(0xffffffffu, bin);
          if (valid && (threadIdx.x & 31) == __ffs(same) - 1)
            atomicAdd(&sh_hist[bin], (uint32_t)__popc(same));
        } else if (valid) {
          atomicAdd(&sh_hist[key >> 20], 1u);
        }
      }
    }
  }
  if (HIST) {
    __syncthreads();
    uint32_t* gh = a.hist + tl * kHistBins;
    for (int b = threadIdx.x; b < kHistBins; b += kScoreThreads) {
      const uint32_t v = sh_hist[b];
      if (v) atomicAdd(gh + b, v);
    }
  }
}

// ---------------------------------------------------------------------------
// shared helpers of the select kernels (1024 threads)
// ---------------------------------------------------------------------------
constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;

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

// Bin holding the `need`-th largest element of a histogram of `nbins` bins
// (nbins a multiple of kSelThreads): sets *bin and *above (elements in higher
// bins) and returns true.  If the histogram holds fewer than `need` elements
// (inconsistent scratch) it returns false with *bin = 0 and *above = 0, so that
// every later index stays in range.  Every thread must call it.
__device__ __forceinline__ bool find_bin(const int* hist, int nbins, int need, int* warp_sums,
                                         uint32_t* s_bin, int* s_above, int* s_ok) {
  if (threadIdx.x == 0) {
    *s_bin = 0u;
    *s_above = 0;
    *s_ok = 0;
  }
  const int per = nbins / kSelThreads;
  // thread i owns ranks [i*per, (i+1)*per) counted from the top bin down
  int c = 0;
  for (int r = 0; r < per; ++r) c += hist[nbins - 1 - (threadIdx.x * per + r)];
  int tot;
  int before = block_exclusive_scan(c, warp_sums, tot);   // syncs order the defaults first
  for (int r = 0; r < per; ++r) {
    const int b = nbins - 1 - (threadIdx.x * per + r);
    const int h = hist[b];
    if (before < need && before + h >= need) {
      *s_bin = (uint32_t)b;
      *s_above = before;
      *s_ok = 1;
    }
    before += h;
  }
  __syncthreads();
  return *s_ok != 0;
}

// ---------------------------------------------------------------------------
// decode-mode selection: one CTA per query, keys in global (L2) memory
// ---------------------------------------------------------------------------
constexpr int kCandCap = 4096;
constexpr int kWarpCap = kCandCap / 32;   // candidate slice of one warp
constexpr int kBatch = 16;   // independent L2 loads in flight per thread

__global__ void __launch_bounds__(kSelThreads) topk_select_bitmap_kernel(SelectArgs a) {
  // dynamic: candidate keys [kCandCap], candidate ids [kCandCap], selection
  // bitmap [W], tie bitmap [W]
  extern __shared__ uint32_t dsm[];
  __shared__ int hist[kHistBins];
  uint32_t* cand_key = dsm;
  int32_t* cand_idx = reinterpret_cast<int32_t*>(dsm + kCandCap);
  __shared__ int warp_sums[32];
  __shared__ uint32_t s_bin;
  __shared__ int s_above, s_ok, s_overflow;
  __shared__ int s_wcnt[kSelWarps];

  const int64_t tl = blockIdx.x;
  const int64_t t = a.t_begin + tl;
  const int64_t pos = a.q_pos ? a.q_pos[t] : t;
  const int64_t n = min(pos / a.m, a.max_entries);
  const int k = a.top_k;
  int32_t* idx = a.idx_out + t * k;
  float* sco = a.score_out ? a.score_out + t * k : nullptr;
  const uint32_t* keys = a.keys + tl * a.key_stride;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (n <= k) {
    for (int64_t j = tid; j < k; j += kSelThreads) {
      idx[j] = j < n ? (int32_t)j : -1;
      if (sco) sco[j] = j < n ? key_score(keys[j]) : -INFINITY;
    }
    if (tid == 0) a.count_out[t] = (int32_t)n;
    return;
  }
  const int W = (int)((n + 31) >> 5);
  uint32_t* sel = dsm + 2 * kCandCap;
  uint32_t* tie = sel + W;

  // level 1: the 12-bit histogram built while scoring
  {
    uint32_t hv[kHistBins / kSelThreads];
#pragma unroll
    for (int i = 0; i < kHistBins / kSelThreads; ++i) hv[i] = a.hist[tl * kHistBins + tid + i * kSelThreads];
#pragma unroll
    for (int i = 0; i < kHistBins / kSelThreads; ++i) hist[tid + i * kSelThreads] = (int)hv[i];
  }
  __syncthreads();
  bool consistent = find_bin(hist, kHistBins, k, warp_sums, &s_bin, &s_above, &s_ok);
  uint32_t prefix = s_bin << 20, mask = 0xfff00000u;
  int need = k - s_above;
  int cnt = hist[s_bin];
  int shift = 20;
  __syncthreads();
  // refine the prefix by one 10-bit digit with a pass over the keys
  auto refine = [&]() {
    shift -= 10;
    for (int b = tid; b < 1024; b += kSelThreads) hist[b] = 0;
    __syncthreads();
    for (int64_t base = tid; base < n; base += kBatch * kSelThreads) {
      uint32_t kk[kBatch];
#pragma unroll
      for (int e = 0; e < kBatch; ++e) {
        const int64_t j = base + (int64_t)e * kSelThreads;
        kk[e] = j < n ? keys[j] : 0u;
      }
#pragma unroll
      for (int e = 0; e < kBatch; ++e) {
        const int64_t j = base + (int64_t)e * kSelThreads;
        if (j < n && (kk[e] & mask) == prefix) atomicAdd(&hist[(kk[e] >> shift) & 1023u], 1);
      }
    }
    __syncthreads();
    consistent &= find_bin(hist, 1024, need, warp_sums, &s_bin, &s_above, &s_ok);
    prefix |= s_bin << shift;
    mask |= 1023u << shift;
    need -= s_above;
    cnt = hist[s_bin];
    __syncthreads();
  };
  while (cnt > kCandCap && shift > 0) refine();
  // one pass: bitmap of keys above the prefix; keys equal to it are
  // candidates, appended to the warp's own slice with a running count held
  // in registers (no shared counter); a slice overflow refines the prefix by
  // another digit and repeats the pass
  for (;;) {
    if (tid == 0) s_overflow = 0;
    __syncthreads();
    int wcnt = 0;
    for (int wb = warp; wb < W; wb += kBatch * kSelWarps) {
      uint32_t kk[kBatch];
#pragma unroll
      for (int e = 0; e < kBatch; ++e) {
        const int64_t j = (int64_t)(wb + e * kSelWarps) * 32 + lane;
        kk[e] = j < n ? keys[j] : 0u;
      }
#pragma unroll
      for (int e = 0; e < kBatch; ++e) {
        const int w = wb + e * kSelWarps;
        if (w >= W) break;   // warp-uniform
        const int64_t j = (int64_t)w * 32 + lane;
        const uint32_t mk = kk[e] & mask;
        const bool gt = j < n && mk > prefix;
        const bool eq = j < n && mk == prefix;
        const uint32_t bg = __ballot_sync(0xffffffffu, gt);
        const uint32_t be = __ballot_sync(0xffffffffu, eq);
        if (lane == 0) {
          sel[w] = bg;
          tie[w] = shift == 0 ? be : 0u;
        }
        if (shift > 0 && be) {
          if (eq) {
            const int p = wcnt + __popc(be & ((1u << lane) - 1u));
            if (p < kWarpCap) {
              cand_key[warp * kWarpCap + p] = kk[e];
              cand_idx[warp * kWarpCap + p] = (int32_t)j;
            }
          }
          wcnt += __popc(be);
        }
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
    // candidate c lives in warp slice c / kWarpCap; valid below that slice's count
    auto cand_ok = [&](int c) { return (c % kWarpCap) < s_wcnt[c / kWarpCap]; };
    int nc = 0;
    for (int w = 0; w < kSelWarps; ++w) nc += min(s_wcnt[w], kWarpCap);
    if (need >= nc) {
      for (int c = tid; c < kCandCap; c += kSelThreads)
        if (cand_ok(c)) atomicOr(&sel[cand_idx[c] >> 5], 1u << (cand_idx[c] & 31));
      need = 0;
    } else {
      // radix select of the need-th largest candidate over the low `shift` bits
      uint32_t cp = prefix, cm = mask;
      while (shift > 0) {
        const int dig = shift >= 10 ? 10 : shift;
        shift -= dig;
        const uint32_t dm = (1u << dig) - 1u;
        for (int b = tid; b < 1024; b += kSelThreads) hist[b] = 0;
        __syncthreads();
        for (int c = tid; c < kCandCap; c += kSelThreads)
          if (cand_ok(c) && (cand_key[c] & cm) == cp) atomicAdd(&hist[(cand_key[c] >> shift) & dm], 1);
        __syncthreads();
        consistent &= find_bin(hist, 1024, need, warp_sums, &s_bin, &s_above, &s_ok);
        cp |= s_bin << shift;
        cm |= dm << shift;
        need -= s_above;
        __syncthreads();
      }
      // cp is the k-th largest key; `need` of its copies are still to take
      for (int c = tid; c < kCandCap; c += kSelThreads) {
        if (!cand_ok(c)) continue;
        const uint32_t key = cand_key[c];
        const int j = cand_idx[c];
        if (key > cp) atomicOr(&sel[j >> 5], 1u << (j & 31));
        else if (key == cp) atomicOr(&tie[j >> 5], 1u << (j & 31));
      }
    }
  }
  __syncthreads();
  // ties: the first `need` set bits of tie[] in index order
  const int wpt = (W + kSelThreads - 1) / kSelThreads;
  const int w0 = tid * wpt, w1 = min(W, w0 + wpt);
  int c = 0;
  for (int w = w0; w < w1; ++w) c += __popc(tie[w]);
  int tot;
  int before = block_exclusive_scan(c, warp_sums, tot);
  for (int w = w0; w < w1; ++w) {
    uint32_t x = tie[w];
    const int pc = __popc(x);
    int take = need - before;
    take = take < 0 ? 0 : (take > pc ? pc : take);
    uint32_t kept = 0;
    for (int i = 0; i < take; ++i) {
      const uint32_t low = x & (0u - x);
      kept |= low;
      x ^= low;
    }
    sel[w] |= kept;
    before += pc;
  }
  __syncthreads();
  // ascending compaction of the selection bitmap
  c = 0;
  for (int w = w0; w < w1; ++w) c += __popc(sel[w]);
  int o = block_exclusive_scan(c, warp_sums, tot);
  for (int w = w0; w < w1; ++w) {
    uint32_t x = sel[w];
    while (x) {
      const int b = __ffs(x) - 1;
      x &= x - 1;
      if (o < k) {
        const int64_t j = (int64_t)w * 32 + b;
        idx[o] = (int32_t)j;
        if (sco) sco[o] = key_score(keys[j]);
      }
      ++o;
    }
  }
  if (tid == 0) {
    a.count_out[t] = k;
    if (!consistent) report(a.err, kErrSelect, (int32_t)t, k);
  }
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

template <int CI, int NT, bool HIST>
cudaError_t launch_score(const Launch& L, const IndexerArgs& a, int64_t t_count) {
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, indexer_score_kernel<CI, NT, HIST>,
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
  indexer_score_kernel<CI, NT, HIST><<<grid, kScoreThreads, 0, L.stream>>>(a, chunk);
  return cudaSuccess;
}

}  // namespace

bool select_uses_bitmap(int64_t t_count, int64_t max_entries) {
  return t_count <= kBitmapSelectMaxQueries && max_entries <= kBitmapSelectMaxEntries;
}

cudaError_t launch_indexer_scores(const Launch& L, const IndexerArgs& a, int64_t t_count) {
  if (t_count == 0 || a.max_entries == 0) return cudaSuccess;
  if (a.fp4) return launch_indexer_scores_fp4(L, a, t_count);
#ifndef CSA_NO_TC_INDEXER
  if (tc_indexer_prefill_supported(a, t_count)) return launch_indexer_scores_tc_prefill(L, a, t_count);
  if (tc_indexer_supported(a, t_count)) return launch_indexer_scores_tc(L, a, t_count);
#endif
  const int nt = (a.H_I + 7) / 8;
  const int ntb = nt <= 1 ? 1 : nt <= 2 ? 2 : nt <= 4 ? 4 : 8;
  const bool hist = a.hist != nullptr;
  L.begin(kKernelIndexerScore);
#define CSA_SCORE_CASE(CI_, NT_)                                                        \
  if (a.c_I == CI_ && ntb == NT_) {                                                     \
    if (hist) launch_score<CI_, NT_, true>(L, a, t_count);                      \
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
  if (a.hist != nullptr) {
    const int W = (int)((a.max_entries + 31) / 32);
    const size_t bytes = (size_t)(2 * kCandCap + 2 * W) * sizeof(uint32_t);
    cudaFuncSetAttribute(topk_select_bitmap_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (2 * kCandCap + 2 * (int)(kBitmapSelectMaxEntries / 32)) * (int)sizeof(uint32_t));
    topk_select_bitmap_kernel<<<(unsigned)t_count, kSelThreads, bytes, L.stream>>>(a);
  } else {
    const size_t bytes = (size_t)((a.max_entries + 3) & ~int64_t(3)) * sizeof(uint32_t);   // whole uint4 stores
    cudaFuncSetAttribute(topk_select_radix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kRadixSelectMaxEntries * (int)sizeof(uint32_t));
    topk_select_radix_kernel<<<(unsigned)t_count, kSelThreads, bytes, L.stream>>>(a);
  }
  return L.end(kKernelTopkSelect);
}

}  // namespace csa
