// Step 2 on tcgen05 tensor cores: lightning-indexer scores streamed from HBM.
//
// DeepSeek-V4 book, Ch.6 "The lightning indexer": I[t,s] = sum_h w[t,h] *
// ReLU(qI[t,h] . K[s]) over the eligible s < floor(t/m).
//
// Persistent kernel, one CTA per SM, three roles:
//   warp 0     TMA producer: items of 256 keys of one query (one 256-row
//              box, or four 64-row boxes for a paged cache; 128-byte swizzle)
//              plus the query's head rows, into a
//              6-stage shared-memory ring (one mbarrier per stage and
//              direction);
//   warp 1     allocates TMEM and issues tcgen05.mma: two M = 128 key tiles
//              per item against the indexer heads (padded to NH = 16, 32 or
//              64) on N, key dim c_I = 64 or 128 as K in steps of 16, into
//              one of four 2 NH-column TMEM sets;
//   warps 2-9  epilogue, two groups of four warps taking alternate items:
//              tcgen05.ld of their 32 TMEM lanes (one key per tile), ReLU,
//              the head-weighted sum, the order-preserving score key, and the
//              fused selection's filter: keys that reach the query's threshold
//              are appended to its candidate list (one atomic per warp); no
//              other score leaves the SM.
// The valid (query, 256-key chunk) pairs are numbered through a prefix sum
// over the queries' chunk counts; the producers of all CTAs take them two at a
// time from one launch-wide counter, so SMs that stream faster take more (on
// B200 some SMs see ~20% less bandwidth than others).  The producer passes
// each item's query, chunk and head weights to the MMA warp and the epilogue
// through a 16-entry ring with its own full / empty barriers.  Every wait is
// bounded; a timeout is reported in the workspace header.
#include "kernels.h"
#include "lowprec.cuh"
#include "tc.cuh"

namespace csa {

namespace {

constexpr int kTileRows = 128;                     // MMA M
constexpr int kItemRows = 2 * kTileRows;           // keys per pipeline item
constexpr int kBoxRows = 64;                       // TMA box height (page granule)
constexpr int kKeyTileBytes = kTileRows * 128;     // 64 bf16 per row
constexpr int kStageKeyBytes = 2 * kKeyTileBytes;
constexpr int kEpiWarps = 8;                       // two groups of four
constexpr int kThreads = (2 + kEpiWarps) * 32;

// Decode-mode layout for key dim CI (64 or 128) and NH padded heads: an
// item's keys are CI / 64 column blocks of kItem rows x 128 bytes (256-row TMA
// boxes of the 128-byte swizzle), the query's heads as many blocks of NH rows.
// An item is 512 keys for CI = 64 (the issuing threads' work per item is
// mostly fixed, so larger items stream closer to the memory bound) and 256
// for CI = 128 (so that several stages still fit).
template <int CI, int NH>
struct ScoreCfg {
  static constexpr int kItem = CI == 64 ? 512 : 256;
  static constexpr int kTiles = kItem / kTileRows;
  static constexpr int kKB = CI / 64;
  static constexpr int kKeyBlk = kItem * 128;
  static constexpr int kStageKey = kKB * kKeyBlk;
  static constexpr int kQBlk = NH * 128;
  static constexpr int kQBytes = kKB * kQBlk;
  // as many stages as fit beside the kernel's static shared memory (<= 6)
  static constexpr int kFit = (205 * 1024) / (kStageKey + kQBytes);
  static constexpr int kStages = kFit < 6 ? kFit : 6;
  static constexpr int kAccCols = kTiles * NH;     // kTiles key tiles of NH columns
  static constexpr int kAccSets = 4 * kAccCols <= 512 ? 4 : 2;   // TMEM accumulator sets
  static constexpr int kTmemCols = kAccSets * kAccCols <= 128 ? 128 : kAccSets * kAccCols <= 256 ? 256 : 512;
  static constexpr uint32_t kIdesc = tc::idesc_bf16(128, NH);
  static constexpr int kSmem = kStages * (kStageKey + kQBytes) + 1024;
  static_assert(kAccSets * kAccCols <= 512 && kStages >= 2, "decode scorer layout");
};
constexpr int kMaxQueries = 2048;
constexpr int kRing = 16;                          // item metadata ring (> stages + accumulator sets)
constexpr int kGrab = 2;                           // items taken from the work counter at once
#ifndef CSA_SCORE_STATIC_PCT
#define CSA_SCORE_STATIC_PCT 70
#endif
constexpr int kStaticPct = CSA_SCORE_STATIC_PCT;   // items dealt out statically, percent

// What the producer tells the MMA warp and the epilogue about item j: the
// query (-1 ends the stream), the 256-key chunk and the query's head weights.
struct __align__(16) ItemMeta {
  float w[64];
  int32_t t, chunk, pad0, pad1;
};

struct TcIndexerParams {
  IndexerArgs a;
  int64_t t_count;
};

__device__ __forceinline__ int64_t eligible(const IndexerArgs& a, int64_t t) {
  const int64_t pos = a.q_pos ? __ldg(a.q_pos + t) : t;
  const int64_t n = pos / a.m;
  return n < a.max_entries ? n : a.max_entries;
}

template <int CI, int NH>
__global__ void __launch_bounds__(kThreads, 1)
indexer_score_tc_kernel(const __grid_constant__ CUtensorMap tmap_keys,
                        const __grid_constant__ CUtensorMap tmap_q, TcIndexerParams p) {
  using Cfg = ScoreCfg<CI, NH>;
  constexpr int kStages = Cfg::kStages, kTmemCols = Cfg::kTmemCols, kAcc = Cfg::kAccSets;
  pdl_trigger();
  const IndexerArgs& a = p.a;
  const int T = (int)p.t_count;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages];
  __shared__ __align__(8) uint64_t tfull_bar[kAcc], tempty_bar[kAcc];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int32_t prefix[kMaxQueries + 1];
  __shared__ int32_t nelig[kMaxQueries];
  __shared__ ItemMeta ring[kRing];
  __shared__ __align__(8) uint64_t ring_full[kRing], ring_empty[kRing];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t keys_sm = base;                                // kStages x kStageKey
  const uint32_t q_sm = base + kStages * Cfg::kStageKey;        // kStages x kQBytes

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(smem_u32(&full_bar[i]), 1);
      mbar_init(smem_u32(&empty_bar[i]), 1);
    }
    for (int i = 0; i < kAcc; ++i) {
      mbar_init(smem_u32(&tfull_bar[i]), 1);
      mbar_init(smem_u32(&tempty_bar[i]), 4);
    }
    for (int i = 0; i < kRing; ++i) {
      mbar_init(smem_u32(&ring_full[i]), 1);
      mbar_init(smem_u32(&ring_empty[i]), 5);   // the MMA warp + one epilogue group
    }
    mbar_fence_init();
  }
  if (warp == 1) tc::tmem_alloc(smem_u32(&tmem_base_sh), kTmemCols);
  // chunk counts and their exclusive prefix (warp 0; T <= kMaxQueries)
  if (warp == 0) {
    const int per = (T + 31) / 32;
    const int t0 = lane * per, t1 = min(T, t0 + per);
    int32_t sum = 0;
    for (int t = t0; t < t1; ++t) {
      const int64_t pos = a.q_pos ? __ldg(a.q_pos + a.t_begin + t) : a.t_begin + t;
      if (pos / a.m > a.max_entries && blockIdx.x == 0)
        report(a.err, kErrEligible, (int32_t)(a.t_begin + t), pos / a.m);
      const int64_t n = eligible(a, a.t_begin + t);
      nelig[t] = (int32_t)n;
      // queries that take all of their entries are not scored
      prefix[t] = n <= a.skip_le ? 0 : (int32_t)((n + Cfg::kItem - 1) / Cfg::kItem);
      sum += prefix[t];
    }
    int32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int32_t run = incl - sum;
    for (int t = t0; t < t1; ++t) {
      const int32_t c = prefix[t];
      prefix[t] = run;
      run += c;
    }
    if (lane == 31) prefix[T] = incl;
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem_base = tmem_base_sh;
  const int32_t V = prefix[T];

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tc::prefetch_tmap(&tmap_keys);
      tc::prefetch_tmap(&tmap_q);
      int64_t issued = 0;
      bool ok = true;
      // Items come from the work counter kGrab at a time; the grab after the
      // current one is requested as soon as the current one starts, and the
      // next item's query and head weights load while this item's keys are
      // issued, so neither latency sits between two items.
      // The first kStaticPct percent of the items are dealt out statically
      // (a contiguous range per CTA, streamed in order); the rest go through
      // the work counter.
      const int32_t Vs = (int32_t)((int64_t)V * kStaticPct / 100);
      const int32_t s_lo = (int32_t)((int64_t)Vs * blockIdx.x / gridDim.x);
      const int32_t s_hi = (int32_t)((int64_t)Vs * (blockIdx.x + 1) / gridDim.x);
      int32_t g_next = s_lo < s_hi ? s_lo : Vs + (int32_t)atomicAdd(a.work, (uint32_t)kGrab);
      bool in_static = s_lo < s_hi;
      int32_t nxt = 0, lim = 0;
      int tq = 0;
      auto take = [&]() -> int32_t {
        if (nxt >= lim) {
          if (g_next >= V) return -1;
          nxt = g_next;
          if (in_static) {
            lim = s_hi;
            in_static = false;
          } else {
            lim = g_next + kGrab < V ? g_next + kGrab : V;
          }
          g_next = Vs + (int32_t)atomicAdd(a.work, (uint32_t)kGrab);
          int l = 0, r = T;   // the query: last tq with prefix[tq] <= nxt
          while (r - l > 1) {
            const int mid = (l + r) >> 1;
            if (prefix[mid] <= nxt) l = mid; else r = mid;
          }
          tq = l;
        }
        while (prefix[tq + 1] <= nxt) ++tq;
        return nxt++;
      };
      float wreg[NH];
      int32_t seq_reg = 0;
      int w_tq = -1;
      auto load_w = [&]() {   // the query's head weights and sequence
        if (tq == w_tq) return;
        w_tq = tq;
        const int64_t t = a.t_begin + tq;
#pragma unroll
        for (int h = 0; h < NH; ++h) wreg[h] = h < a.H_I ? __ldg(a.w + t * a.H_I + h) : 0.f;
        seq_reg = a.seq_id ? __ldg(a.seq_id + t) : 0;
      };
      int32_t item = take();
      if (item >= 0) load_w();
      while (item >= 0) {
        const int32_t chunk = item - prefix[tq];
        const int64_t t = a.t_begin + tq;
        const int64_t s0 = (int64_t)chunk * Cfg::kItem;
        const int rs = (int)(issued % kRing);
        if (!mbar_wait(smem_u32(&ring_empty[rs]), (uint32_t)(((issued / kRing) & 1) ^ 1))) {
          report(a.err, kErrTimeout, (int32_t)t, 16);
          ok = false;
          break;
        }
#pragma unroll
        for (int h = 0; h < NH; ++h) ring[rs].w[h] = wreg[h];
        ring[rs].t = tq;
        ring[rs].chunk = chunk;
        mbar_arrive(smem_u32(&ring_full[rs]));
        const int cur_tq = tq;
        const int32_t seq = seq_reg;
        const int slot = (int)(issued % kStages);
        if (!mbar_wait(smem_u32(&empty_bar[slot]), (uint32_t)(((issued / kStages) & 1) ^ 1))) {
          report(a.err, kErrTimeout, (int32_t)t, 10);
          ok = false;
          break;
        }
        const uint32_t fb = smem_u32(&full_bar[slot]);
        mbar_arrive_expect_tx(fb, Cfg::kStageKey + Cfg::kQBytes);
        const uint32_t kst = keys_sm + slot * Cfg::kStageKey;
        if (a.keys.page_table == nullptr) {
          // contiguous: 256-row boxes per column block
#pragma unroll
          for (int kb = 0; kb < Cfg::kKB; ++kb)
#pragma unroll
            for (int hh = 0; hh < Cfg::kItem / kItemRows; ++hh)
              tc::tma_load_2d(kst + kb * Cfg::kKeyBlk + hh * kItemRows * 128, &tmap_keys, 64 * kb,
                              (int32_t)((int64_t)seq * a.keys.seq_stride + s0 + hh * kItemRows), fb);
        } else {
#pragma unroll
        for (int h = 0; h < Cfg::kItem / kBoxRows; ++h) {
          const int64_t s = s0 + h * kBoxRows;
          int64_t row;
          {
            const int64_t pi = s / a.keys.page_size;
            const int32_t page = pi < a.keys.max_pages
                                     ? __ldg(a.keys.page_table + (int64_t)seq * a.keys.max_pages + pi)
                                     : -1;
            row = (int64_t)page * a.keys.page_size + (s - pi * a.keys.page_size);
            if (page < 0 || row >= a.keys.n_rows) {
              if (s < nelig[cur_tq]) report(a.err, kErrPageId, (int32_t)t, page);
              row = 0;
            }
          }
#pragma unroll
          for (int kb = 0; kb < Cfg::kKB; ++kb)
            tc::tma_load_2d(kst + kb * Cfg::kKeyBlk + h * kBoxRows * 128, &tmap_keys, 64 * kb,
                            (int32_t)row, fb);
        }
        }
#pragma unroll
        for (int kb = 0; kb < Cfg::kKB; ++kb)
          tc::tma_load_2d(q_sm + slot * Cfg::kQBytes + kb * Cfg::kQBlk, &tmap_q, 64 * kb,
                          (int32_t)(t * a.H_I), fb);
        ++issued;
        item = take();
        if (item >= 0) load_w();
      }
      // two end markers: the MMA warp stops at the first, each epilogue
      // group (alternate items) at the one that falls to it
      for (int e = 0; ok && e < 2; ++e) {
        const int64_t j = issued + e;
        const int rs = (int)(j % kRing);
        if (!mbar_wait(smem_u32(&ring_empty[rs]), (uint32_t)(((j / kRing) & 1) ^ 1))) {
          report(a.err, kErrTimeout, 0, 17);
          break;
        }
        ring[rs].t = -1;
        mbar_arrive(smem_u32(&ring_full[rs]));
      }
      // every copy must land before the CTA can exit: the last kStages
      // issued stages hold the latest phase of every slot
      const int64_t first = issued > kStages ? issued - kStages : 0;
      for (int64_t d = first; d < issued; ++d)
        mbar_wait(smem_u32(&full_bar[d % kStages]), (uint32_t)((d / kStages) & 1), 200000000ll);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      for (int64_t j = 0;; ++j) {
        const int rs = (int)(j % kRing);
        if (!mbar_wait(smem_u32(&ring_full[rs]), (uint32_t)((j / kRing) & 1))) {
          report(a.err, kErrTimeout, (int32_t)j, 18);
          break;
        }
        const bool end = ring[rs].t < 0;
        mbar_arrive(smem_u32(&ring_empty[rs]));
        if (end) break;
        const int slot = (int)(j % kStages);
        const int acc = (int)(j % kAcc);
        if (!mbar_wait(smem_u32(&full_bar[slot]), (uint32_t)((j / kStages) & 1))) {
          report(a.err, kErrTimeout, (int32_t)j, 11);
          break;
        }
        if (!mbar_wait(smem_u32(&tempty_bar[acc]), (uint32_t)(((j / kAcc) & 1) ^ 1))) {
          report(a.err, kErrTimeout, (int32_t)j, 12);
          break;
        }
        tc::fence_after_sync();
        const uint32_t qa = q_sm + slot * Cfg::kQBytes;
#pragma unroll
        for (int h = 0; h < Cfg::kTiles; ++h) {
#pragma unroll
          for (int kb = 0; kb < Cfg::kKB; ++kb) {
            const uint32_t ka = keys_sm + slot * Cfg::kStageKey + kb * Cfg::kKeyBlk + h * kKeyTileBytes;
#pragma unroll
            for (int k = 0; k < 4; ++k)
              tc::mma_bf16_ss(tmem_base + acc * Cfg::kAccCols + h * NH, tc::smem_desc_sw128(ka + 32 * k),
                              tc::smem_desc_sw128(qa + kb * Cfg::kQBlk + 32 * k), Cfg::kIdesc,
                              kb > 0 || k > 0);
          }
        }
        tc::mma_commit(smem_u32(&empty_bar[slot]));   // smem stage free when the MMAs finish
        tc::mma_commit(smem_u32(&tfull_bar[acc]));    // accumulators ready
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // the thresholds and zeroed counts come from the sample pass, which may
    // still be running when this kernel starts (the producer and the MMA warp
    // do not need them)
    pdl_wait();
    const int ew = warp - 2;
    const int group = ew >> 2;                 // handles items j with j % 2 == group
    const int quarter = warp & 3;              // TMEM lanes this warp may read
    const int row = quarter * 32 + lane;       // key within a 128-key tile
    int t_cached = -1;
    int64_t n_elig = 0;
    uint32_t tau = 0;
    CandidateBatch<Cfg::kTiles> pend;   // the previous item's candidates, stored after this item's atomic
    for (int64_t j = group;; j += 2) {
      const int rs = (int)(j % kRing);
      if (!mbar_wait(smem_u32(&ring_full[rs]), (uint32_t)((j / kRing) & 1))) {
        if (lane == 0) report(a.err, kErrTimeout, (int32_t)j, 19);
        break;
      }
      const int tq = ring[rs].t;
      const int32_t chunk = ring[rs].chunk;
      float wv[NH];
#pragma unroll
      for (int h = 0; h < NH; h += 4) {
        const float4 w4 = *reinterpret_cast<const float4*>(&ring[rs].w[h]);
        wv[h] = w4.x;
        wv[h + 1] = w4.y;
        wv[h + 2] = w4.z;
        wv[h + 3] = w4.w;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ring_empty[rs]));
      if (tq < 0) break;
      const int acc = (int)(j % kAcc);
      if (tq != t_cached) {
        t_cached = tq;
        n_elig = nelig[tq];
        tau = __ldg(a.tau + tq);
      }
      if (!mbar_wait(smem_u32(&tfull_bar[acc]), (uint32_t)((j / kAcc) & 1))) {
        if (lane == 0) report(a.err, kErrTimeout, (int32_t)j, 13);
        break;
      }
      tc::fence_after_sync();
      // this key's ReLU-weighted head sum in each tile, NH columns each, 16
      // columns per TMEM load, every tile's load of a column group before one wait
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * Cfg::kAccCols;
      float scs[Cfg::kTiles];
#pragma unroll
      for (int h = 0; h < Cfg::kTiles; ++h) scs[h] = 0.f;
#pragma unroll
      for (int c = 0; c < NH / 16; ++c) {
        uint32_t r[Cfg::kTiles][16];
#pragma unroll
        for (int h = 0; h < Cfg::kTiles; ++h) tc::tmem_ld16(taddr + h * NH + 16 * c, r[h]);
        tc::tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < Cfg::kTiles; ++h)
#pragma unroll
          for (int k = 0; k < 16; ++k) scs[h] = fmaf(wv[16 * c + k], fmaxf(__uint_as_float(r[h][k]), 0.f), scs[h]);
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tempty_bar[acc]));
      const int64_t s0 = (int64_t)chunk * Cfg::kItem;
      bool pass[Cfg::kTiles];
      uint32_t keys[Cfg::kTiles], ents[Cfg::kTiles];
#pragma unroll
      for (int h = 0; h < Cfg::kTiles; ++h) {
        const float sc = scs[h];
        const int64_t s = s0 + h * kTileRows + row;
        keys[h] = score_key(sc);
        ents[h] = (uint32_t)s;
        pass[h] = s < n_elig && keys[h] >= tau;
      }
      CandidateBatch<Cfg::kTiles> cur;
      cur.issue(a, tq, pass, keys, ents);
      pend.flush(a);
      pend = cur;
    }
    pend.flush(a);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 1) tc::tmem_dealloc(tmem_base, kTmemCols);
}

// ---------------------------------------------------------------------------
// Many-query mode: every query reads the same sequence (prefill), so a block
// of QB = 128 / H_I consecutive queries shares each key tile.  The block's
// (query, head) rows fill the MMA N side (128), keys the M side: one 256-key
// item is two 128 x 128 x 64 products into 256 TMEM columns, 16x fewer key
// reads per score than the one-query decode mode.  The epilogue thread owns
// a key and sums the ReLU-weighted heads of each query of the block from its
// own TMEM row, so no cross-thread reduction is needed.  Items (block, chunk)
// follow the same hybrid static / work-counter schedule as decode mode.
// Two passes use it (no score matrix is stored):
//   MODE kPSample: only the block's sampled chunks (psample_chunk); every key
//     goes to the query's sample row psample[t, i * 256 + key];
//   MODE kPFused: every chunk; keys that reach the query's tau are appended to
//     its candidate list, one slot reservation per warp and query.
// ---------------------------------------------------------------------------
constexpr int kPStages = 4;
constexpr int kPQTileBytes = 128 * 128;                  // 128 rows x 64 bf16
constexpr int kPStageBytes = kStageKeyBytes + kPQTileBytes;
constexpr int kPAcc = 2;                                 // one per epilogue group
constexpr int kPTmemCols = 512;
constexpr uint32_t kPIdesc = tc::idesc_bf16(128, 128);
constexpr int kMaxBlocks = 2048;
constexpr int kPRing = 16;
constexpr int kPEpiWarps = 16;                 // four groups: (item parity, key tile)
constexpr int kPThreads = (2 + kPEpiWarps) * 32;

struct __align__(16) BlockMeta {
  float w[128];       // the block's head weights in (query, head) order
  int32_t nel[32];    // eligible entries of each of the block's queries (0 past the chunk)
  uint32_t tau[32];   // their candidate thresholds (fused pass)
  int32_t b, chunk, sidx, pad1;   // sidx: the chunk's ordinal among the sampled ones
};

constexpr int kPSample = 1, kPFused = 2;

template <int HI, int MODE>
__global__ void __launch_bounds__(kPThreads, 1)
indexer_score_tc_prefill_kernel(const __grid_constant__ CUtensorMap tmap_keys,
                                const __grid_constant__ CUtensorMap tmap_q, TcIndexerParams p) {
  const IndexerArgs& a = p.a;
  const int T = (int)p.t_count;
  constexpr int QB = 128 / HI;
  const int NB = (T + QB - 1) / QB;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kPStages], empty_bar[kPStages];
  __shared__ __align__(8) uint64_t tfull_bar[kPAcc], tempty_bar[kPAcc];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int32_t prefix[kMaxBlocks + 1];
  __shared__ int32_t bmin[MODE == kPSample ? kMaxBlocks : 1];   // fewest eligible entries per block
  __shared__ BlockMeta ring[kPRing];
  __shared__ __align__(8) uint64_t ring_full[kPRing], ring_empty[kPRing];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;   // kPStages x (32 + 16) KB

  if (threadIdx.x == 0) {
    for (int i = 0; i < kPStages; ++i) {
      mbar_init(smem_u32(&full_bar[i]), 1);
      mbar_init(smem_u32(&empty_bar[i]), 1);
    }
    for (int i = 0; i < kPAcc; ++i) {
      mbar_init(smem_u32(&tfull_bar[i]), 1);
      mbar_init(smem_u32(&tempty_bar[i]), 8);   // the two groups reading the set
    }
    for (int i = 0; i < kPRing; ++i) {
      mbar_init(smem_u32(&ring_full[i]), 1);
      mbar_init(smem_u32(&ring_empty[i]), 9);   // the MMA warp + two epilogue groups
    }
    mbar_fence_init();
  }
  // items per block: fused pass, the chunks of its longest query that is
  // scored; sample pass, its sampled chunks (from its fewest and most
  // eligible entries)
  for (int b = threadIdx.x; b < NB; b += kPThreads) {
    prefix[b] = 0;
    if (MODE == kPSample) bmin[b] = INT32_MAX;
  }
  if (warp == 1) tc::tmem_alloc(smem_u32(&tmem_base_sh), kPTmemCols);
  __syncthreads();
  for (int t = threadIdx.x; t < T; t += kPThreads) {
    const int64_t pos = a.q_pos ? __ldg(a.q_pos + a.t_begin + t) : a.t_begin + t;
    if (MODE == kPFused && pos / a.m > a.max_entries && blockIdx.x == 0)
      report(a.err, kErrEligible, (int32_t)(a.t_begin + t), pos / a.m);
    const int64_t n = eligible(a, a.t_begin + t);
    if (MODE == kPSample) {
      atomicMax(&prefix[t / QB], (int32_t)n);
      atomicMin(&bmin[t / QB], (int32_t)n);
    } else if (n > a.skip_le) {
      atomicMax(&prefix[t / QB], (int32_t)((n + kItemRows - 1) / kItemRows));
    }
  }
  __syncthreads();
  if (MODE == kPSample)
    for (int b = threadIdx.x; b < NB; b += kPThreads)
      prefix[b] = psample_chunks(bmin[b], prefix[b], a.cand_cap, a.skip_le);
  __syncthreads();
  if (warp == 0) {   // exclusive prefix over the blocks
    const int per = (NB + 31) / 32;
    const int b0 = lane * per, b1 = min(NB, b0 + per);
    int32_t sum = 0;
    for (int b = b0; b < b1; ++b) sum += prefix[b];
    int32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int32_t run = incl - sum;
    for (int b = b0; b < b1; ++b) {
      const int32_t c = prefix[b];
      prefix[b] = run;
      run += c;
    }
    if (lane == 31) prefix[NB] = incl;
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem_base = tmem_base_sh;
  const int32_t V = prefix[NB];

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // The whole warp: lane 0 takes items, waits and issues the copies; the
    // lanes fill the ring entry together (one float4 of weights and at most
    // one query length each).
    if (lane == 0) {
      tc::prefetch_tmap(&tmap_keys);
      tc::prefetch_tmap(&tmap_q);
    }
    int64_t issued = 0;
    bool ok = true;
    const int32_t Vs = (int32_t)((int64_t)V * kStaticPct / 100);
    const int32_t s_lo = (int32_t)((int64_t)Vs * blockIdx.x / gridDim.x);
    const int32_t s_hi = (int32_t)((int64_t)Vs * (blockIdx.x + 1) / gridDim.x);
    int32_t g_next = 0;
    if (lane == 0) g_next = s_lo < s_hi ? s_lo : Vs + (int32_t)atomicAdd(a.work, (uint32_t)kGrab);
    bool in_static = s_lo < s_hi;
    int32_t nxt = 0, lim = 0;
    int bq = 0, bq_meta = -1;
    // lane 0's view of the item sequence (the other lanes receive it by shuffle)
    auto take = [&]() -> int32_t {
      if (nxt >= lim) {
        if (g_next >= V) return -1;
        nxt = g_next;
        if (in_static) {
          lim = s_hi;
          in_static = false;
        } else {
          lim = g_next + kGrab < V ? g_next + kGrab : V;
        }
        g_next = Vs + (int32_t)atomicAdd(a.work, (uint32_t)kGrab);
        int l = 0, r = NB;   // the block: last bq with prefix[bq] <= nxt
        while (r - l > 1) {
          const int mid = (l + r) >> 1;
          if (prefix[mid] <= nxt) l = mid; else r = mid;
        }
        bq = l;
      }
      while (prefix[bq + 1] <= nxt) ++bq;
      return nxt++;
    };
    for (;;) {
      int32_t item = -1;
      if (lane == 0) item = take();
      item = __shfl_sync(0xffffffffu, item, 0);
      const int b_now = __shfl_sync(0xffffffffu, bq, 0);
      if (item < 0) break;
      const int32_t sidx = item - prefix[b_now];
      const int32_t chunk = MODE == kPSample
                                ? (int32_t)psample_chunk(sidx, prefix[b_now + 1] - prefix[b_now], bmin[b_now])
                                : sidx;
      const int64_t t0 = (int64_t)b_now * QB;           // first query of the block (chunk-local)
      const int64_t s0 = (int64_t)chunk * kItemRows;
      const int rs = (int)(issued % kPRing);
      bool got = true;
      if (lane == 0) got = mbar_wait(smem_u32(&ring_empty[rs]), (uint32_t)(((issued / kPRing) & 1) ^ 1));
      __syncwarp();
      if (!__shfl_sync(0xffffffffu, got, 0)) {
        if (lane == 0) report(a.err, kErrTimeout, (int32_t)(a.t_begin + t0), 16);
        ok = false;
        break;
      }
      BlockMeta& mt = ring[rs];
      const int64_t nq = T - t0 < QB ? T - t0 : QB;
      if (b_now != bq_meta) {
        // the block's weights (128 consecutive floats, 16-byte aligned) and lengths
        const float4* wsrc = reinterpret_cast<const float4*>(a.w + (a.t_begin + t0) * HI);
        reinterpret_cast<float4*>(mt.w)[lane] =
            lane * 4 < nq * HI ? __ldg(wsrc + lane) : make_float4(0.f, 0.f, 0.f, 0.f);
        if (lane < QB) {
          mt.nel[lane] = lane < nq ? (int32_t)eligible(a, a.t_begin + t0 + lane) : 0;
          mt.tau[lane] = MODE == kPFused && lane < nq ? __ldg(a.tau + t0 + lane) : 0u;
        }
        bq_meta = b_now;
      } else {
        const BlockMeta& pm = ring[(issued - 1) % kPRing];
        reinterpret_cast<float4*>(mt.w)[lane] = reinterpret_cast<const float4*>(pm.w)[lane];
        if (lane < QB) {
          mt.nel[lane] = pm.nel[lane];
          mt.tau[lane] = pm.tau[lane];
        }
      }
      if (lane == 0) {
        mt.b = b_now;
        mt.chunk = chunk;
        mt.sidx = sidx;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ring_full[rs]));   // releases the lanes' writes (after the warp sync)
      if (lane == 0) {
        const int slot = (int)(issued % kPStages);
        if (!mbar_wait(smem_u32(&empty_bar[slot]), (uint32_t)(((issued / kPStages) & 1) ^ 1))) {
          report(a.err, kErrTimeout, (int32_t)(a.t_begin + t0), 10);
          got = false;
        } else {
          const uint32_t fb = smem_u32(&full_bar[slot]);
          const uint32_t st = base + slot * kPStageBytes;
          mbar_arrive_expect_tx(fb, kPStageBytes);
          if (a.keys.page_table == nullptr) {
            tc::tma_load_2d(st, &tmap_keys, 0, (int32_t)s0, fb);
          } else {
#pragma unroll
            for (int h = 0; h < kItemRows / kBoxRows; ++h) {
              const int64_t s = s0 + h * kBoxRows;
              const int64_t pi = s / a.keys.page_size;
              const int32_t page = pi < a.keys.max_pages ? __ldg(a.keys.page_table + pi) : -1;
              int64_t row = (int64_t)page * a.keys.page_size + (s - pi * a.keys.page_size);
              if (page < 0 || row >= a.keys.n_rows) {
                if (s < mt.nel[0] || s < mt.nel[QB - 1]) report(a.err, kErrPageId, (int32_t)(a.t_begin + t0), page);
                row = 0;
              }
              tc::tma_load_2d(st + h * kBoxRows * 128, &tmap_keys, 0, (int32_t)row, fb);
            }
          }
          tc::tma_load_2d(st + kStageKeyBytes, &tmap_q, 0, (int32_t)((a.t_begin + t0) * HI), fb);
        }
      }
      if (!__shfl_sync(0xffffffffu, got, 0)) {
        ok = false;
        break;
      }
      ++issued;
    }
    if (lane == 0) {
      for (int e = 0; ok && e < 2; ++e) {   // end markers, as in decode mode
        const int64_t j = issued + e;
        const int rs = (int)(j % kPRing);
        if (!mbar_wait(smem_u32(&ring_empty[rs]), (uint32_t)(((j / kPRing) & 1) ^ 1))) {
          report(a.err, kErrTimeout, 0, 17);
          break;
        }
        ring[rs].b = -1;
        mbar_arrive(smem_u32(&ring_full[rs]));
      }
      const int64_t first = issued > kPStages ? issued - kPStages : 0;
      for (int64_t d = first; d < issued; ++d)
        mbar_wait(smem_u32(&full_bar[d % kPStages]), (uint32_t)((d / kPStages) & 1), 200000000ll);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      for (int64_t j = 0;; ++j) {
        const int rs = (int)(j % kPRing);
        if (!mbar_wait(smem_u32(&ring_full[rs]), (uint32_t)((j / kPRing) & 1))) {
          report(a.err, kErrTimeout, (int32_t)j, 18);
          break;
        }
        const bool end = ring[rs].b < 0;
        mbar_arrive(smem_u32(&ring_empty[rs]));
        if (end) break;
        const int slot = (int)(j % kPStages);
        const int acc = (int)(j % kPAcc);
        if (!mbar_wait(smem_u32(&full_bar[slot]), (uint32_t)((j / kPStages) & 1)) ||
            !mbar_wait(smem_u32(&tempty_bar[acc]), (uint32_t)(((j / kPAcc) & 1) ^ 1))) {
          report(a.err, kErrTimeout, (int32_t)j, 11);
          break;
        }
        tc::fence_after_sync();
        const uint32_t st = base + slot * kPStageBytes;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc::mma_bf16_ss(tmem_base + acc * 256 + h * 128, tc::smem_desc_sw128(st + h * kKeyTileBytes + 32 * k),
                            tc::smem_desc_sw128(st + kStageKeyBytes + 32 * k), kPIdesc, k > 0);
        }
        tc::mma_commit(smem_u32(&empty_bar[slot]));
        tc::mma_commit(smem_u32(&tfull_bar[acc]));
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int eg = (warp - 2) >> 2;            // 0..3
    const int group = eg >> 1;                 // items j with j % 2 == group, accumulator set `group`
    const int h = eg & 1;                      // the key tile of the item this group scores
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;       // key within a 128-key tile
    constexpr int qpc = 32 / HI;               // queries per 32 TMEM columns
    for (int64_t j = group;; j += 2) {
      const int rs = (int)(j % kPRing);
      if (!mbar_wait(smem_u32(&ring_full[rs]), (uint32_t)((j / kPRing) & 1))) {
        if (lane == 0) report(a.err, kErrTimeout, (int32_t)j, 19);
        break;
      }
      const BlockMeta& mt = ring[rs];
      const int bq = mt.b;
      if (bq < 0) {
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&ring_empty[rs]));
        break;
      }
      const int acc = group;
      if (!mbar_wait(smem_u32(&tfull_bar[acc]), (uint32_t)((j / kPAcc) & 1))) {
        if (lane == 0) report(a.err, kErrTimeout, (int32_t)j, 13);
        break;
      }
      tc::fence_after_sync();
      const int64_t s0 = (int64_t)mt.chunk * kItemRows;
      const int64_t t0 = (int64_t)bq * QB;
      {
        const int64_t s = s0 + h * kTileRows + row;
        const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * 256 + h * 128;
        uint32_t keys[QB];   // this thread's key for each query of the block
#pragma unroll
        for (int c = 0; c < 4; ++c) {   // 32 (query, head) columns at a time
          uint32_t r0[16], r1[16];
          tc::tmem_ld16(taddr + c * 32, r0);
          tc::tmem_ld16(taddr + c * 32 + 16, r1);
          tc::tmem_wait_ld();
          float x[32], wq[32];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            x[i] = fmaxf(__uint_as_float(r0[i]), 0.f);
            x[16 + i] = fmaxf(__uint_as_float(r1[i]), 0.f);
          }
#pragma unroll
          for (int i = 0; i < 32; i += 4) {   // this chunk's 32 head weights
            const float4 w4 = *reinterpret_cast<const float4*>(&mt.w[c * 32 + i]);
            wq[i] = w4.x;
            wq[i + 1] = w4.y;
            wq[i + 2] = w4.z;
            wq[i + 3] = w4.w;
          }
#pragma unroll
          for (int qq = 0; qq < qpc; ++qq) {
            float sc = 0.f;
#pragma unroll
            for (int hh = 0; hh < HI; ++hh) sc = fmaf(wq[qq * HI + hh], x[qq * HI + hh], sc);
            keys[c * qpc + qq] = score_key(sc);
          }
        }
        if (MODE == kPSample) {
          // the sampled chunks are readable by every query of the block
          const int64_t col = (int64_t)mt.sidx * kItemRows + h * kTileRows + row;
#pragma unroll
          for (int q = 0; q < QB; ++q)
            if (t0 + q < T) a.psample[(t0 + q) * kPSampleKeys + col] = keys[q];
        } else {
          // candidates: one ballot per query; lane q reserves the warp's slots
          // for query q, so that all the block's reservations are one round trip
          uint32_t mym = 0u;
#pragma unroll
          for (int q = 0; q < QB; ++q) {
            const int32_t nq = mt.nel[q];
            const uint32_t m = __ballot_sync(0xffffffffu, s < nq && nq > a.skip_le && keys[q] >= mt.tau[q]);
            if (lane == q) mym = m;
          }
          const uint32_t mybase = mym ? atomicAdd(a.cand_count + t0 + lane, (uint32_t)__popc(mym)) : 0u;
#pragma unroll
          for (int q = 0; q < QB; ++q) {
            const uint32_t m = __shfl_sync(0xffffffffu, mym, q);
            const uint32_t b0 = __shfl_sync(0xffffffffu, mybase, q);
            if ((m >> lane) & 1u) {
              const uint32_t slot = b0 + (uint32_t)__popc(m & ((1u << lane) - 1u));
              if (slot < (uint64_t)a.cand_cap)
                a.cand[(t0 + q) * a.cand_cap + slot] = make_uint2(keys[q], (uint32_t)s);
            }
          }
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&tempty_bar[acc]));
        mbar_arrive(smem_u32(&ring_empty[rs]));
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 1) tc::tmem_dealloc(tmem_base, kPTmemCols);
}

// ---------------------------------------------------------------------------
// 4-bit keys (few-query mode): the same persistent pipeline as the bf16
// decode scorer, on block-scaled tensor-core MMAs
// (tcgen05.mma.kind::mxf4.block_scale, M = 128 keys, K = 64 per instruction):
// the tensor cores apply both scales, so TMEM holds the exact scaled dot
// products.  An item's key codes (E2M1, 32 bytes per 64-dim block) and scale
// bytes arrive by 1-D bulk copies (a TMA box of 32-byte rows streams at a
// fraction of the rate).  The MMA reads operands in the 32-byte-swizzled
// K-major layout, where rows 4..7 of every 8 have their two 16-byte halves
// exchanged:
//  * 64-dim keys land as stored and are read as if swizzled, so those rows
//    reach the MMA with halves exchanged; the B operand holds every head twice,
//    as stored (columns 0 .. NH) and with halves exchanged (NH .. 2 NH), each
//    key's scale bytes are exchanged to match, and the epilogue takes each row's
//    dot products from the copy that pairs its halves correctly;
//  * 128-dim keys are moved into the swizzled layout by the MMA warp's lanes.
// The producer warp quantizes each query's heads (the block quantizer of
// csa_quantize_mxfp4) once and writes them, with their scale bytes, into the
// stage; the MMA warp arranges the keys' scale bytes in the layout tcgen05.cp
// moves to TMEM and one lane issues the MMAs.  The epilogue is the bf16
// scorer's.  A sample mode (MODE kFp4Sample) scores only psample_chunks whole
// chunks of each query and writes their keys to psample.
// ---------------------------------------------------------------------------
constexpr int kFp4Sample = 1, kFp4Fused = 2;
constexpr int kFMinItem = 256;                 // the smallest item (keys) of any shape

template <int CI, int NH, bool SAMPLE>
struct Fp4Cfg {
  static constexpr bool kSwap = CI == 64;                 // codes used as stored (see above)
  static constexpr int kN = kSwap ? 2 * NH : NH;          // MMA N: B rows
  // keys per item (128-key tiles): as many as TMEM holds accumulators for
  // (the per-item work of the producer and MMA warps is mostly fixed); the
  // sample pass takes 256-key chunks
  static constexpr int kItem = SAMPLE || !kSwap ? 256 : kN <= 32 ? 1024 : kN == 64 ? 512 : 256;
  static constexpr int kTiles = kItem / kTileRows;
  static constexpr int kKB = CI / 64;                     // 64-element blocks per key (one MMA each)
  static constexpr int kCodeBlk = kItem * 32;             // one block of an item's key codes
  static constexpr int kCodes = kKB * kCodeBlk;
  static constexpr int kQBlk = kN * 32;
  static constexpr int kQCodes = kKB * kQBlk;
  static constexpr int kRawSc = kItem * (CI / 32);        // the keys' scale bytes as stored
  static constexpr int kSfa = kTiles * kKB * 512;         // per (tile, block): 32 rows x 16 B
  static constexpr int kSfb = kKB * 512;
  // a query's operand image (B codes, then its SFB blocks): one bulk copy
  static constexpr int kQImg = kQCodes + kSfb;
  static constexpr int kQOff = kCodes;
  static constexpr int kSfbOff = kQOff + kQCodes;
  static constexpr int kRawOff = kSfbOff + kSfb;
  static constexpr int kSfaOff = kRawOff + kRawSc;
  // where the copied codes land: the operand itself (kSwap), else a staging area
  static constexpr int kRawCodes = kSwap ? 0 : kItem * (CI / 2);
  static constexpr int kRawCOff = kSwap ? 0 : (kSfaOff + kSfa + 127) / 128 * 128;
  static constexpr int kStage = ((kSwap ? kSfaOff + kSfa : kRawCOff + kRawCodes) + 1023) / 1024 * 1024;
  static constexpr int kStages = (200 * 1024) / kStage < 8 ? (200 * 1024) / kStage : 8;
  static constexpr int kAccCols = kTiles * kN;
  // per set: SFA kTiles x kKB, then one SFB copy per issuing warp (kKB each), 4 columns each
  static constexpr int kSfCols = 4 * (kTiles + 2) * kKB;
  static constexpr int kAccF = 2 * (kAccCols + kSfCols) <= 512 ? 2 : 1;   // accumulator sets
  static constexpr int kSfBase = kAccF * kAccCols;
  static constexpr int kTmemCols = 512;
  static constexpr uint32_t kIdesc = tc::idesc_mxf4(128, kN);
  static constexpr int kSmem = kStages * kStage + 1024;
  static_assert(kN % 16 == 0 && kN <= 128 && NH >= 8, "MMA N");
  static_assert(kQImg <= kFp4ImgSlots * 8, "query image");
  static_assert(kSfBase + kAccF * kSfCols <= kTmemCols, "TMEM columns");
};

// An item's rows in 64-row runs (pages, or the end of a contiguous cache):
// lane 0 sets the barrier's byte count and issues bulk copies of the codes
// (any row count) and of the scale bytes of whole multiples of 8 rows; lanes
// 1 .. 31 load a run's last (rows mod 8) scale bytes themselves.  Rows past
// the cache's end are not copied (they are never scored valid).
template <int CI, int ITEM>
__device__ __noinline__ void fp4_copy_runs(CacheRef keys, const uint8_t* k_scales, WsHeader* err,
                                           uint32_t codes_sm, uint32_t scales_sm, uint8_t* scales_p,
                                           uint32_t fb, int32_t seq, int64_t s0, int64_t n_cur, int32_t t,
                                           int lane) {
  constexpr int kRuns = ITEM / kBoxRows, cb = CI / 2, nsc = CI / 32;
  const uint8_t* const kc = reinterpret_cast<const uint8_t*>(keys.data);
  int64_t row0[kRuns];
  int nrow[kRuns];
  uint32_t bytes = 0;
#pragma unroll
  for (int hb = 0; hb < kRuns; ++hb) {
    const int64_t s = s0 + hb * kBoxRows;
    int64_t row;
    if (keys.page_table == nullptr) {
      row = (int64_t)seq * keys.seq_stride + s;
    } else {
      const int64_t pi = s / keys.page_size;
      const int32_t page = pi < keys.max_pages ? __ldg(keys.page_table + (int64_t)seq * keys.max_pages + pi) : -1;
      row = (int64_t)page * keys.page_size + (s - pi * keys.page_size);
      if (page < 0 || row >= keys.n_rows) {
        if (lane == 0 && s < n_cur) report(err, kErrPageId, t, page);
        row = 0;
      }
    }
    int64_t nr = keys.n_rows - row;
    nr = nr < 0 ? 0 : (nr > kBoxRows ? kBoxRows : nr);
    row0[hb] = row;
    nrow[hb] = (int)nr;
    bytes += (uint32_t)(nrow[hb] * cb + (nrow[hb] & ~7) * nsc);
  }
  if (lane == 0) {
    mbar_arrive_expect_tx(fb, bytes);
#pragma unroll
    for (int hb = 0; hb < kRuns; ++hb) {
      if (nrow[hb] > 0)
        bulk_g2s(codes_sm + hb * kBoxRows * cb, kc + row0[hb] * cb, (uint32_t)(nrow[hb] * cb), fb);
      if ((nrow[hb] & ~7) > 0)
        bulk_g2s(scales_sm + hb * kBoxRows * nsc, k_scales + row0[hb] * nsc, (uint32_t)((nrow[hb] & ~7) * nsc), fb);
    }
  } else {
    bool wrote = false;
    const int sl = lane - 1;
#pragma unroll
    for (int hb = 0; hb < kRuns; ++hb) {
      const int nb = nrow[hb] & ~7;
      if (sl < (nrow[hb] - nb) * nsc) {
        const int r = nb + sl / nsc, jj = sl % nsc;
        scales_p[(hb * kBoxRows + r) * nsc + jj] = k_scales[(row0[hb] + r) * nsc + jj];
        wrote = true;
      }
    }
    if (wrote) fence_async_smem_cta();
  }
}

// One warp per query: the block quantizer of csa_quantize_mxfp4 on each head
// (zero codes for the padded heads), then the stage image of the MMA's B
// operand: B row r = head r mod NH (rows NH .. 2 NH with halves exchanged when
// kSwap) in the K-major 32-byte swizzle, and the SFB blocks in the tcgen05.cp
// layout (row r at byte 4 (r / 32) + k of row r mod 32).
template <int CI, int NH>
__global__ void __launch_bounds__(128) fp4_query_image_kernel(IndexerArgs a, int64_t t_count) {
  using Cfg = Fp4Cfg<CI, NH, false>;
  __shared__ __align__(16) uint8_t codes[4][NH * CI / 2];
  __shared__ uint8_t sfs[4][NH * CI / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (blockIdx.x == 0 && threadIdx.x == 0) *a.work = 0u;
  const int64_t tl = (int64_t)blockIdx.x * 4 + warp;
  if (tl >= t_count) return;
  const int64_t t = a.t_begin + tl;
  for (int b = lane; b < NH * (CI / 32); b += 32) {
    const int h = b / (CI / 32), v = b - h * (CI / 32);
    uint32_t w4[4] = {0u, 0u, 0u, 0u};
    uint32_t sb = 0u;
    if (h < a.H_I) sb = lowprec::quantize_block(a.q_idx + (t * a.H_I + h) * CI + 32 * v, w4);
    *reinterpret_cast<uint4*>(codes[warp] + h * (CI / 2) + 16 * v) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    sfs[warp][h * (CI / 32) + v] = (uint8_t)sb;
  }
  __syncwarp();
  uint8_t* const img = a.q_img + tl * Cfg::kQImg;
#pragma unroll
  for (int kb = 0; kb < Cfg::kKB; ++kb) {
    for (int c = lane; c < Cfg::kN * 2; c += 32) {
      const int r = c >> 1, half = c & 1, hh = r & (NH - 1), xs = Cfg::kSwap && r >= NH;
      *reinterpret_cast<uint4*>(img + kb * Cfg::kQBlk + r * 32 + (((half ^ (r >> 2)) & 1) << 4)) =
          *reinterpret_cast<const uint4*>(codes[warp] + hh * (CI / 2) + kb * 32 + (half ^ xs) * 16);
    }
    const int m0 = lane;
    uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int cc = 0; cc < (Cfg::kN + 31) / 32; ++cc) {
      const int r = m0 + 32 * cc, hh = r & (NH - 1), xs = Cfg::kSwap && r >= NH;
      if (r < Cfg::kN)
        w[cc] = (uint32_t)sfs[warp][hh * (CI / 32) + 2 * kb + xs] |
                ((uint32_t)sfs[warp][hh * (CI / 32) + 2 * kb + (xs ^ 1)] << 8);
    }
    *reinterpret_cast<uint4*>(img + Cfg::kQCodes + kb * 512 + m0 * 16) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// producer, MMA issuer, kEpiWarps epilogue warps, the operand warp, a second
// MMA issuer (the two take alternate halves of an item's tiles)
constexpr int kFThreads = kThreads + 64;
constexpr int kOpWarp = kThreads / 32;
constexpr int kMma2Warp = kOpWarp + 1;

template <int CI, int NH, int MODE>
__global__ void __launch_bounds__(kFThreads, 1)
indexer_score_fp4_tc_kernel(TcIndexerParams p) {
  using Cfg = Fp4Cfg<CI, NH, MODE == kFp4Sample>;
  constexpr int kStages = Cfg::kStages, kAccF = Cfg::kAccF;
  pdl_trigger();   // the next launch may set itself up; it waits for this one's results
  const IndexerArgs& a = p.a;
  const int T = (int)p.t_count;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[kStages], empty_bar[kStages], opnd_bar[kStages];
  __shared__ __align__(8) uint64_t tfull_bar[kAccF], tempty_bar[kAccF];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int32_t prefix[kMaxQueries + 1];
  __shared__ int32_t nelig[kMaxQueries];
  __shared__ ItemMeta ring[kRing];
  __shared__ __align__(8) uint64_t ring_full[kRing], ring_empty[kRing];
  __shared__ __align__(16) float qc_w[NH];                    // the current query's head weights
  __shared__ int32_t slot_q[Cfg::kStages];                   // the query whose heads a stage holds

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - smem_u32(smem_raw));

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      slot_q[i] = -1;
      mbar_init(smem_u32(&full_bar[i]), 2);   // the copies' arrival + the query staging's
      mbar_init(smem_u32(&empty_bar[i]), 2);   // both MMA issuers' commits
      mbar_init(smem_u32(&opnd_bar[i]), 1);   // the operand warp's arrival
    }
    for (int i = 0; i < kAccF; ++i) {
      mbar_init(smem_u32(&tfull_bar[i]), 2);   // both MMA issuers' commits
      mbar_init(smem_u32(&tempty_bar[i]), 4);
    }
    for (int i = 0; i < kRing; ++i) {
      mbar_init(smem_u32(&ring_full[i]), 1);
      mbar_init(smem_u32(&ring_empty[i]), 7);   // two MMA issuers, one epilogue group, the operand warp
    }
    mbar_fence_init();
  }
  if (warp == 1) tc::tmem_alloc(smem_u32(&tmem_base_sh), Cfg::kTmemCols);
  if (warp == 0) {
    // items per query: its chunks (fused pass) or its sampled chunks
    const int per = (T + 31) / 32;
    const int t0 = lane * per, t1 = min(T, t0 + per);
    int32_t sum = 0;
    for (int t = t0; t < t1; ++t) {
      const int64_t pos = a.q_pos ? __ldg(a.q_pos + a.t_begin + t) : a.t_begin + t;
      if (MODE == kFp4Fused && pos / a.m > a.max_entries && blockIdx.x == 0)
        report(a.err, kErrEligible, (int32_t)(a.t_begin + t), pos / a.m);
      const int64_t n = eligible(a, a.t_begin + t);
      nelig[t] = (int32_t)n;
      prefix[t] = MODE == kFp4Sample ? psample_chunks(n, n, a.cand_cap, a.skip_le) * 256 / Cfg::kItem
                                     : (n <= a.skip_le ? 0 : (int32_t)((n + Cfg::kItem - 1) / Cfg::kItem));
      sum += prefix[t];
    }
    int32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int32_t run = incl - sum;
    for (int t = t0; t < t1; ++t) {
      const int32_t c = prefix[t];
      prefix[t] = run;
      run += c;
    }
    if (lane == 31) prefix[T] = incl;
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem_base = tmem_base_sh;
  const int32_t V = prefix[T];

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // the work counter and the query images come from the preceding launch,
    // which may still run while this kernel sets itself up
    pdl_wait();
    int64_t issued = 0;
    bool ok = true;
    const int32_t Vs = (int32_t)((int64_t)V * kStaticPct / 100);
    const int32_t s_lo = (int32_t)((int64_t)Vs * blockIdx.x / gridDim.x);
    const int32_t s_hi = (int32_t)((int64_t)Vs * (blockIdx.x + 1) / gridDim.x);
    int32_t g_next = 0;
    if (lane == 0) g_next = s_lo < s_hi ? s_lo : Vs + (int32_t)atomicAdd(a.work, (uint32_t)kGrab);
    bool in_static = s_lo < s_hi;
    int32_t nxt = 0, lim = 0;
    int tq = 0, q_tq = -1;
    int32_t q_seq = 0;
    auto take = [&]() -> int32_t {   // lane 0's view of the item sequence
      if (nxt >= lim) {
        if (g_next >= V) return -1;
        nxt = g_next;
        if (in_static) {
          lim = s_hi;
          in_static = false;
        } else {
          lim = g_next + kGrab < V ? g_next + kGrab : V;
        }
        g_next = Vs + (int32_t)atomicAdd(a.work, (uint32_t)kGrab);
        int l = 0, r = T;
        while (r - l > 1) {
          const int mid = (l + r) >> 1;
          if (prefix[mid] <= nxt) l = mid; else r = mid;
        }
        tq = l;
      }
      while (prefix[tq + 1] <= nxt) ++tq;
      return nxt++;
    };
    const int nsc = CI / 32;   // scale bytes per key row
    const uint8_t* const kc = reinterpret_cast<const uint8_t*>(a.keys.data);   // CI / 2 code bytes per row
    for (;;) {
      int32_t item = -1;
      if (lane == 0) item = take();
      item = __shfl_sync(0xffffffffu, item, 0);
      const int cur = __shfl_sync(0xffffffffu, tq, 0);
      if (item < 0) break;
      const int32_t sidx = item - prefix[cur];
      const int64_t n_cur = nelig[cur];
      const int32_t chunk = MODE == kFp4Sample
                                ? (int32_t)(((2 * (int64_t)sidx + 1) * (n_cur / Cfg::kItem)) /
                                            (2 * (int64_t)(prefix[cur + 1] - prefix[cur])))
                                : sidx;
      const int64_t t = a.t_begin + cur;
      const int64_t s0 = (int64_t)chunk * Cfg::kItem;
      if (cur != q_tq) {
        for (int h = lane; h < NH; h += 32) qc_w[h] = h < a.H_I ? __ldg(a.w + t * a.H_I + h) : 0.f;
        q_tq = cur;
        q_seq = a.seq_id ? __ldg(a.seq_id + t) : 0;
        __syncwarp();
      }
      const int32_t seq = q_seq;
      const int rs = (int)(issued % kRing);
      const int slot = (int)(issued % kStages);
      bool got = true;
      if (lane == 0) {
        got = mbar_wait_susp(smem_u32(&ring_empty[rs]), (uint32_t)(((issued / kRing) & 1) ^ 1));
        if (!got) report(a.err, kErrTimeout, (int32_t)t, 16);
      }
      if (!__shfl_sync(0xffffffffu, got, 0)) {
        ok = false;
        break;
      }
      for (int h = lane; h < NH; h += 32) ring[rs].w[h] = qc_w[h];
      __syncwarp();
      if (lane == 0) {
        ring[rs].t = cur;
        ring[rs].chunk = MODE == kFp4Sample ? sidx : chunk;
        mbar_arrive(smem_u32(&ring_full[rs]));   // releases the lanes' weights (after the warp sync)
        got = mbar_wait_susp(smem_u32(&empty_bar[slot]), (uint32_t)(((issued / kStages) & 1) ^ 1));
        if (!got) report(a.err, kErrTimeout, (int32_t)t, 10);
      }
      if (!__shfl_sync(0xffffffffu, got, 0)) {
        ok = false;
        break;
      }
      uint8_t* const st = base_ptr + slot * Cfg::kStage;
      const uint32_t sst = base + slot * Cfg::kStage;
      const uint32_t fb = smem_u32(&full_bar[slot]);
      // the item's codes and scale bytes: two bulk copies for a whole item of a
      // contiguous cache, else page by page (out of line)
      const int64_t cbase = (int64_t)seq * a.keys.seq_stride + s0;
      if (a.keys.page_table == nullptr && a.keys.n_rows - cbase >= Cfg::kItem) {
        if (lane == 0) {
          mbar_arrive_expect_tx(fb, (uint32_t)(Cfg::kItem * (CI / 2 + nsc)));
          bulk_g2s(sst + Cfg::kRawCOff, kc + cbase * (CI / 2), (uint32_t)(Cfg::kItem * (CI / 2)), fb);
          bulk_g2s(sst + Cfg::kRawOff, a.k_scales + cbase * nsc, (uint32_t)(Cfg::kItem * nsc), fb);
        }
      } else {
        fp4_copy_runs<CI, Cfg::kItem>(a.keys, a.k_scales, a.err, sst + Cfg::kRawCOff, sst + Cfg::kRawOff,
                                      st + Cfg::kRawOff, fb, seq, s0, n_cur, (int32_t)t, lane);
      }
      // the query's operand image, unless the stage still holds it
      if (lane == 0 && slot_q[slot] != cur) {
        mbar_expect_tx(fb, (uint32_t)Cfg::kQImg);
        bulk_g2s(sst + Cfg::kQOff, a.q_img + (int64_t)cur * Cfg::kQImg, (uint32_t)Cfg::kQImg, fb);
      }
      __syncwarp();
      if (lane == 0) {
        slot_q[slot] = cur;
        mbar_arrive(fb);   // the staging's arrival: releases the lanes' writes
      }
      ++issued;
    }
    if (lane == 0) {
      for (int e = 0; ok && e < 2; ++e) {   // end markers (the MMA warp stops at the first)
        const int64_t j = issued + e;
        const int rs = (int)(j % kRing);
        if (!mbar_wait_susp(smem_u32(&ring_empty[rs]), (uint32_t)(((j / kRing) & 1) ^ 1))) {
          report(a.err, kErrTimeout, 0, 17);
          break;
        }
        ring[rs].t = -1;
        mbar_arrive(smem_u32(&ring_full[rs]));
      }
      const int64_t first = issued > kStages ? issued - kStages : 0;
      for (int64_t d = first; d < issued; ++d)
        mbar_wait(smem_u32(&full_bar[d % kStages]), (uint32_t)((d / kStages) & 1), 200000000ll);
    }
  } else if (warp == 1 || warp == kMma2Warp) {
    // ------------------------------------------------------------ MMA issuers
    // (lane 0 of each issues half of an item's tiles, with its own copy of the
    // query's scale factors; the operand warp has arranged the stage's operands)
    const int half = warp == 1 ? 0 : 1;
    constexpr int kHalf = Cfg::kTiles / 2;
    for (uint32_t j = 0;; ++j) {
      const int rs = (int)(j % kRing);
      bool got = true, end = false;
      if (lane == 0) {
        got = mbar_wait_susp(smem_u32(&ring_full[rs]), (j / kRing) & 1u);
        if (!got) report(a.err, kErrTimeout, (int32_t)j, 18);
        else {
          end = ring[rs].t < 0;
          mbar_arrive(smem_u32(&ring_empty[rs]));
        }
      }
      got = __shfl_sync(0xffffffffu, got, 0);
      end = __shfl_sync(0xffffffffu, end, 0);
      if (!got || end) break;
      const int slot = (int)(j % kStages);
      const int acc = (int)(j % kAccF);
      if (lane == 0) {
        got = mbar_wait_susp(smem_u32(&full_bar[slot]), (j / kStages) & 1u) &&
              mbar_wait_susp(smem_u32(&opnd_bar[slot]), (j / kStages) & 1u) &&
              mbar_wait_susp(smem_u32(&tempty_bar[acc]), ((j / kAccF) & 1u) ^ 1u);
        if (!got) report(a.err, kErrTimeout, (int32_t)j, 11);
        else {
          tc::fence_after_sync();
          const uint32_t sst = base + slot * Cfg::kStage;
          const uint32_t sf = tmem_base + Cfg::kSfBase + acc * Cfg::kSfCols;
          const uint32_t sfb = sf + 4 * (Cfg::kTiles + half) * Cfg::kKB;   // this issuer's SFB copy
#pragma unroll
          for (int i = half * kHalf * Cfg::kKB; i < (half + 1) * kHalf * Cfg::kKB; ++i)
            tc::copy_scales(sf + 4 * i, sst + Cfg::kSfaOff + i * 512);
#pragma unroll
          for (int kb = 0; kb < Cfg::kKB; ++kb) tc::copy_scales(sfb + 4 * kb, sst + Cfg::kSfbOff + kb * 512);
#pragma unroll
          for (int h = half * kHalf; h < (half + 1) * kHalf; ++h)
#pragma unroll
            for (int kb = 0; kb < Cfg::kKB; ++kb)
              tc::mma_mxf4_ss(tmem_base + acc * Cfg::kAccCols + h * Cfg::kN,
                              tc::smem_desc_sw32(sst + kb * Cfg::kCodeBlk + h * 128 * 32),
                              tc::smem_desc_sw32(sst + Cfg::kQOff + kb * Cfg::kQBlk), Cfg::kIdesc,
                              sf + 4 * (h * Cfg::kKB + kb), sfb + 4 * kb, kb > 0);
          tc::mma_commit(smem_u32(&empty_bar[slot]));
          tc::mma_commit(smem_u32(&tfull_bar[acc]));
        }
      }
      if (!__shfl_sync(0xffffffffu, got, 0)) break;
    }
  } else if (warp == kOpWarp) {
    // ------------------------------------------------------------ operands
    // Once a stage's copies land: for 128-dim keys the codes into the K-major
    // 32-byte swizzle (row r of block kb at 32 r, its 16-byte halves exchanged
    // when bit 2 of r is set); then lane m0 writes row m0 of every SFA block
    // (tile h, block kb): bytes 4 c + (0, 1) hold the scale bytes of key
    // m0 + 32 c, exchanged for the rows whose halves the MMA sees exchanged.
    for (uint32_t j = 0;; ++j) {
      const int rs = (int)(j % kRing);
      bool got = true, end = false;
      if (lane == 0) {
        got = mbar_wait_susp(smem_u32(&ring_full[rs]), (j / kRing) & 1u);
        if (!got) report(a.err, kErrTimeout, (int32_t)j, 20);
        else {
          end = ring[rs].t < 0;
          mbar_arrive(smem_u32(&ring_empty[rs]));
        }
      }
      got = __shfl_sync(0xffffffffu, got, 0);
      end = __shfl_sync(0xffffffffu, end, 0);
      if (!got || end) break;
      const int slot = (int)(j % kStages);
      if (lane == 0) {
        got = mbar_wait_susp(smem_u32(&full_bar[slot]), (j / kStages) & 1u);
        if (!got) report(a.err, kErrTimeout, (int32_t)j, 21);
      }
      if (!__shfl_sync(0xffffffffu, got, 0)) break;
      uint8_t* const st = base_ptr + slot * Cfg::kStage;
      if (!Cfg::kSwap) {
        constexpr int kChunks = Cfg::kItem * Cfg::kKB * 2;
        const uint8_t* raw = st + Cfg::kRawCOff;
#pragma unroll 4
        for (int q = lane; q < kChunks; q += 32) {
          const int r = q / (Cfg::kKB * 2), kb = (q >> 1) % Cfg::kKB, half = q & 1;
          const uint4 v = *reinterpret_cast<const uint4*>(raw + r * (CI / 2) + kb * 32 + half * 16);
          *reinterpret_cast<uint4*>(st + kb * Cfg::kCodeBlk + r * 32 + (((half ^ (r >> 2)) & 1) << 4)) = v;
        }
      }
      const int m0 = lane;
      const bool xs = Cfg::kSwap && ((m0 >> 2) & 1);
      const uint16_t* rsc = reinterpret_cast<const uint16_t*>(st + Cfg::kRawOff);
#pragma unroll
      for (int h = 0; h < Cfg::kTiles; ++h)
#pragma unroll
        for (int kb = 0; kb < Cfg::kKB; ++kb) {
          uint32_t w[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint32_t v = rsc[(h * 128 + m0 + 32 * c) * Cfg::kKB + kb];
            w[c] = xs ? ((v >> 8) | ((v & 0xffu) << 8)) : v;
          }
          *reinterpret_cast<uint4*>(st + Cfg::kSfaOff + (h * Cfg::kKB + kb) * 512 + m0 * 16) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
      fence_async_smem_cta();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&opnd_bar[slot]));
    }
  } else {
    // ------------------------------------------------------------ epilogue
    pdl_wait();   // tau and the zeroed candidate counts (fused pass) come from the preceding launch
    const int ew = warp - 2;
    const int group = ew >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    int t_cached = -1;
    int64_t n_elig = 0;
    uint32_t tau = 0;
    CandidateBatch<Cfg::kTiles> pend;
    for (uint32_t j = group;; j += 2) {
      const int rs = (int)(j % kRing);
      if (!mbar_wait_susp(smem_u32(&ring_full[rs]), (j / kRing) & 1u)) {
        if (lane == 0) report(a.err, kErrTimeout, (int32_t)j, 19);
        break;
      }
      const int tq = ring[rs].t;
      const int32_t chunk = ring[rs].chunk;   // the sampled chunk's ordinal in sample mode
      float wv[NH];
#pragma unroll
      for (int h = 0; h < NH; h += 4) {
        const float4 w4 = *reinterpret_cast<const float4*>(&ring[rs].w[h]);
        wv[h] = w4.x;
        wv[h + 1] = w4.y;
        wv[h + 2] = w4.z;
        wv[h + 3] = w4.w;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&ring_empty[rs]));
      if (tq < 0) break;
      const int acc = (int)(j % kAccF);
      if (tq != t_cached) {
        t_cached = tq;
        n_elig = nelig[tq];
        tau = MODE == kFp4Fused ? __ldg(a.tau + tq) : 0u;
      }
      if (!mbar_wait_susp(smem_u32(&tfull_bar[acc]), (uint32_t)((j / kAccF) & 1))) {
        if (lane == 0) report(a.err, kErrTimeout, (int32_t)j, 13);
        break;
      }
      tc::fence_after_sync();
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * Cfg::kAccCols;
      // this row's dot products, from the copy that pairs its halves
      // correctly (columns NH + h for rows 4 .. 7 of every 8 when kSwap, else
      // h), at most 64 columns loaded per wait: kPass passes of kHP heads
      constexpr int kPass = Cfg::kN > 64 ? 2 : 1;
      constexpr int kHP = NH / kPass;
      constexpr int kChN = (kHP + 15) / 16;   // 16-column loads of a pass's plain columns
      const bool second = Cfg::kSwap && ((row >> 2) & 1);
      float scs[Cfg::kTiles];
#pragma unroll
      for (int h = 0; h < Cfg::kTiles; ++h) {
        scs[h] = 0.f;
#pragma unroll
        for (int pa = 0; pa < kPass; ++pa) {
          uint32_t r[4][16];
          const uint32_t tcol = taddr + h * Cfg::kN + pa * kHP;
          if (Cfg::kSwap && kHP < 16) {
            tc::tmem_ld16(tcol, r[0]);   // NH = 8: plain and exchanged copies in one load
          } else {
#pragma unroll
            for (int c = 0; c < kChN; ++c) {
              tc::tmem_ld16(tcol + 16 * c, r[c]);
              if (Cfg::kSwap) tc::tmem_ld16(tcol + NH + 16 * c, r[kChN + c]);
            }
          }
          tc::tmem_wait_ld();
#pragma unroll
          for (int hh = 0; hh < kHP; ++hh) {
            uint32_t v;
            if (Cfg::kSwap && kHP < 16) v = second ? r[0][(8 + hh) & 15] : r[0][hh & 15];
            else if (Cfg::kSwap) v = second ? r[kChN + hh / 16][hh % 16] : r[hh / 16][hh % 16];
            else v = r[hh / 16][hh % 16];
            scs[h] = fmaf(wv[pa * kHP + hh], fmaxf(__uint_as_float(v), 0.f), scs[h]);
          }
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tempty_bar[acc]));
      if (MODE == kFp4Sample) {
#pragma unroll
        for (int h = 0; h < Cfg::kTiles; ++h)
          a.psample[(int64_t)tq * kPSampleKeys + chunk * Cfg::kItem + h * kTileRows + row] = score_key(scs[h]);
        continue;
      }
      const int64_t s0 = (int64_t)chunk * Cfg::kItem;
      bool pass[Cfg::kTiles];
      uint32_t keys[Cfg::kTiles], ents[Cfg::kTiles];
#pragma unroll
      for (int h = 0; h < Cfg::kTiles; ++h) {
        const int64_t s = s0 + h * kTileRows + row;
        keys[h] = score_key(scs[h]);
        ents[h] = (uint32_t)s;
        pass[h] = s < n_elig && keys[h] >= tau;
      }
      CandidateBatch<Cfg::kTiles> cur;
      cur.issue(a, tq, pass, keys, ents);
      pend.flush(a);
      pend = cur;
    }
    if (MODE == kFp4Fused) pend.flush(a);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 1) tc::tmem_dealloc(tmem_base, Cfg::kTmemCols);
}

}  // namespace

bool tc_indexer_supported(const IndexerArgs& a, int64_t t_count) {
  if (a.tau == nullptr) return false;   // fused selection only
  if ((a.c_I != 64 && a.c_I != 128) || a.H_I > 64 || t_count > kMaxQueries) return false;
  if ((a.max_entries + kItemRows - 1) / kItemRows * t_count > INT32_MAX) return false;
  if (a.keys.page_table != nullptr && a.keys.page_size % kBoxRows != 0) return false;
  if (a.keys.n_rows > INT32_MAX || a.T * a.H_I > INT32_MAX) return false;
  if (a.work == nullptr) return false;
  return true;
}

bool tc_indexer_prefill_supported(const IndexerArgs& a, int64_t t_count) {
  if (a.tau == nullptr || a.psample == nullptr || a.fp4) return false;   // the sampled fused selection
  if (a.seq_id != nullptr || a.c_I != 64 || a.work == nullptr) return false;
  if (a.H_I != 4 && a.H_I != 8 && a.H_I != 16) return false;
  // the producer reads a block's 128 head weights as 32 aligned float4
  if ((reinterpret_cast<uintptr_t>(a.w) & 15u) != 0 || ((a.t_begin * a.H_I) & 3) != 0) return false;
  const int64_t qb = 128 / a.H_I;
  const int64_t nb = (t_count + qb - 1) / qb;
  if (nb > kMaxBlocks || (a.max_entries + kItemRows - 1) / kItemRows * nb > INT32_MAX) return false;
  if (a.keys.page_table != nullptr && a.keys.page_size % kBoxRows != 0) return false;
  if (a.keys.n_rows > INT32_MAX || a.T * a.H_I > INT32_MAX) return false;
  return true;
}

cudaError_t launch_indexer_scores_tc_prefill(const Launch& L, const IndexerArgs& a, int64_t t_count,
                                             bool sample) {
  CUtensorMap tk, tq;
  const uint32_t box_rows = a.keys.page_table == nullptr ? kItemRows : kBoxRows;
  if (!make_tmap_bf16_2d(&tk, a.keys.data, 64, (uint64_t)a.keys.n_rows, 64, 64, box_rows))
    return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tq, a.q_idx, 64, (uint64_t)(a.T * a.H_I), 64, 64, 128))
    return cudaErrorInvalidValue;
  TcIndexerParams p;
  p.a = a;
  p.t_count = t_count;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int smem = kPStages * kPStageBytes + 1024;
  L.begin(kKernelIndexerScore);
#define CSA_PREFILL_CASE(H_, M_)                                                                   \
  if (a.H_I == H_ && (M_ == kPSample) == sample) {                                                 \
    cudaFuncSetAttribute(indexer_score_tc_prefill_kernel<H_, M_>,                                  \
                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);                       \
    prefer_max_shared(indexer_score_tc_prefill_kernel<H_, M_>);                                    \
    indexer_score_tc_prefill_kernel<H_, M_><<<(unsigned)sms, kPThreads, smem, L.stream>>>(tk, tq, p); \
  }
  CSA_PREFILL_CASE(4, kPSample)
  CSA_PREFILL_CASE(8, kPSample)
  CSA_PREFILL_CASE(16, kPSample)
  CSA_PREFILL_CASE(4, kPFused)
  CSA_PREFILL_CASE(8, kPFused)
  CSA_PREFILL_CASE(16, kPFused)
#undef CSA_PREFILL_CASE
  return L.end(kKernelIndexerScore);
}

namespace {

template <int CI, int NH>
cudaError_t launch_score_tc(const Launch& L, const IndexerArgs& a, int64_t t_count) {
  using Cfg = ScoreCfg<CI, NH>;
  CUtensorMap tk, tq;
  const uint32_t box_rows = a.keys.page_table == nullptr ? kItemRows : kBoxRows;
  if (!make_tmap_bf16_2d(&tk, a.keys.data, CI, (uint64_t)a.keys.n_rows, CI, 64, box_rows))
    return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tq, a.q_idx, CI, (uint64_t)(a.T * a.H_I), CI, 64, NH))
    return cudaErrorInvalidValue;
  TcIndexerParams p;
  p.a = a;
  p.t_count = t_count;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaFuncSetAttribute(indexer_score_tc_kernel<CI, NH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       Cfg::kSmem);
  prefer_max_shared(indexer_score_tc_kernel<CI, NH>);
  return launch_kernel(indexer_score_tc_kernel<CI, NH>, dim3((unsigned)sms), dim3(kThreads),
                       (size_t)Cfg::kSmem, L.stream, true, tk, tq, p);
}

}  // namespace

bool tc_fp4_indexer_supported(const IndexerArgs& a, int64_t t_count) {
  if (!a.fp4 || a.tau == nullptr || a.psample == nullptr || a.work == nullptr) return false;
  if ((a.c_I != 64 && a.c_I != 128) || a.H_I > 64 || t_count > kMaxQueries) return false;
  if ((a.max_entries + kFMinItem - 1) / kFMinItem * t_count > INT32_MAX) return false;
  if (a.keys.page_table != nullptr && a.keys.page_size % kBoxRows != 0) return false;
  if (a.keys.n_rows > INT32_MAX || a.T * a.H_I > INT32_MAX) return false;
  // code rows and scale-byte copies must stay 16-byte aligned
  const int64_t code_row = a.c_I / 2, sc_row = a.c_I / 32;
  if ((reinterpret_cast<uintptr_t>(a.keys.data) & 15u) || (reinterpret_cast<uintptr_t>(a.k_scales) & 15u))
    return false;
  if (a.keys.page_table == nullptr && ((a.keys.seq_stride * sc_row) % 16 != 0 || (a.keys.seq_stride * code_row) % 16 != 0))
    return false;
  return true;
}

namespace {

template <int CI, int NH, int MODE>
cudaError_t launch_score_fp4_tc(const Launch& L, const IndexerArgs& a, int64_t t_count) {
  using Cfg = Fp4Cfg<CI, NH, MODE == kFp4Sample>;
  TcIndexerParams p;
  p.a = a;
  p.t_count = t_count;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaFuncSetAttribute(indexer_score_fp4_tc_kernel<CI, NH, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       Cfg::kSmem);
  prefer_max_shared(indexer_score_fp4_tc_kernel<CI, NH, MODE>);
  return launch_kernel(indexer_score_fp4_tc_kernel<CI, NH, MODE>, dim3((unsigned)sms), dim3(kFThreads),
                       (size_t)Cfg::kSmem, L.stream, true, p);
}

}  // namespace

cudaError_t launch_fp4_query_images(const Launch& L, const IndexerArgs& a, int64_t t_count) {
  L.begin(kKernelIndexerScore);
  const int nh = a.c_I == 64 && a.H_I <= 8 ? 8 : a.c_I == 64 && a.H_I <= 16 ? 16 : a.H_I <= 32 ? 32 : 64;
  const unsigned grid = (unsigned)((t_count + 3) / 4);
#define CSA_FP4IMG(CI_, NH_) fp4_query_image_kernel<CI_, NH_><<<grid, 128, 0, L.stream>>>(a, t_count);
  if (a.c_I == 64) {
    if (nh == 8) { CSA_FP4IMG(64, 8) } else if (nh == 16) { CSA_FP4IMG(64, 16) }
    else if (nh == 32) { CSA_FP4IMG(64, 32) } else { CSA_FP4IMG(64, 64) }
  } else {
    if (nh == 32) { CSA_FP4IMG(128, 32) } else { CSA_FP4IMG(128, 64) }
  }
#undef CSA_FP4IMG
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return L.end(kKernelIndexerScore);
}

cudaError_t launch_indexer_scores_fp4_tc(const Launch& L, const IndexerArgs& a, int64_t t_count, bool sample) {
  L.begin(kKernelIndexerScore);
  // padded heads: 8 / 16 / 32 / 64 for 64-dim keys (B holds 2 NH rows), 32 / 64 for 128-dim
  const int nh = a.c_I == 64 && a.H_I <= 8 ? 8 : a.c_I == 64 && a.H_I <= 16 ? 16 : a.H_I <= 32 ? 32 : 64;
  cudaError_t e;
#define CSA_FP4TC(CI_, NH_) \
  e = sample ? launch_score_fp4_tc<CI_, NH_, kFp4Sample>(L, a, t_count) : launch_score_fp4_tc<CI_, NH_, kFp4Fused>(L, a, t_count);
  if (a.c_I == 64) {
    if (nh == 8) { CSA_FP4TC(64, 8) } else if (nh == 16) { CSA_FP4TC(64, 16) }
    else if (nh == 32) { CSA_FP4TC(64, 32) } else { CSA_FP4TC(64, 64) }
  } else {
    if (nh == 32) { CSA_FP4TC(128, 32) } else { CSA_FP4TC(128, 64) }
  }
#undef CSA_FP4TC
  if (e != cudaSuccess) return e;
  return L.end(kKernelIndexerScore);
}

cudaError_t launch_indexer_scores_tc(const Launch& L, const IndexerArgs& a, int64_t t_count) {
  L.begin(kKernelIndexerScore);
  const int nh = a.H_I <= 16 ? 16 : a.H_I <= 32 ? 32 : 64;
  cudaError_t e = cudaSuccess;
  if (a.c_I == 64) {
    e = nh == 16 ? launch_score_tc<64, 16>(L, a, t_count)
        : nh == 32 ? launch_score_tc<64, 32>(L, a, t_count) : launch_score_tc<64, 64>(L, a, t_count);
  } else {
    e = nh == 16 ? launch_score_tc<128, 16>(L, a, t_count)
        : nh == 32 ? launch_score_tc<128, 32>(L, a, t_count) : launch_score_tc<128, 64>(L, a, t_count);
  }
  if (e != cudaSuccess) return e;
  return L.end(kKernelIndexerScore);
}

}  // namespace csa
