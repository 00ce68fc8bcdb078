// Step 4 on tcgen05 tensor cores: shared-KV attention over gathered rows.
//
// DeepSeek-V4 book, Ch.6 "Shared key-value MQA" (every head reads the same
// rows, each both key and value) and Ch.7 "The 128-token uncompressed sliding
// window" (selected entries and window rows share one softmax), "Dense
// attention over heavily compressed history", "Learned attention sinks".
//
// Rows sit on the MMA M dimension and heads on N, so one 128-row tile of the
// shared KV feeds both products without a transpose:
//   S^T [128 rows x 64 heads] = KV [128 x 128 dims] . Q^T      (A K-major)
//   O^T [128 dims x 64 heads] += KV^T [dims x rows] . P^T       (A and B MN-major)
// The gathered tile is stored once in the 128-byte swizzled layout; read as a
// K-major operand it is KV, read as an MN-major operand it is KV^T.  P^T is
// written by the softmax threads (thread = row, 64 heads = one 128-byte row).
//
// Warp roles (persistent CTAs over (query, split, head group) work items):
//   warps 9-15 producers: selected rows gathered with 16-byte cp.async into
//              their swizzled slots (through the page table when paged),
//              contiguous rows (HCA, window) with 128-row TMA boxes; the
//              item's query heads once per item
//   warp 8     TMEM allocation and tcgen05.mma issue
//   warps 0-7  online softmax in two warpgroups that split the 64 heads of
//              every tile (thread = row of S^T): per-head tile maxima with
//              redux.sync, a lazily rescaled running max (O^T is rescaled in
//              TMEM only when a head's max grows by more than 2^8), exp2,
//              per-thread partial row sums, bf16 P^T to shared memory; at the
//              end of an item the epilogue (thread = dim of O^T) writes the
//              normalised output or the split partials.
// The kernel may start while the previous kernel on the stream finishes
// (programmatic dependent launch): it sets up its barriers and TMEM and then
// waits for that kernel before it reads anything.
// Every wait is bounded (the workspace header records a timeout).
#include <cmath>

#include "kernels.h"
#include "lowprec.cuh"
#include "tc.cuh"

namespace csa {

namespace {

constexpr int kD = 128;
constexpr int kNP = 64;                         // heads per CTA (MMA N)
constexpr int kRows = 128;                      // rows per tile (MMA M of S^T)
#ifndef CSA_ATTN_STAGES
#define CSA_ATTN_STAGES 4
#endif
constexpr int kStages = CSA_ATTN_STAGES;
constexpr int kKvTile = kRows * kD * 2;         // 32 KB: two 64-dim blocks of 16 KB
constexpr int kKBlock = kRows * 128;            // 16 KB
constexpr int kQTile = kNP * kD * 2;            // 16 KB: two 64-dim blocks of 8 KB
constexpr int kPTile = kRows * kNP * 2;         // 16 KB
#ifndef CSA_ATTN_GROUPS
#define CSA_ATTN_GROUPS 2
#endif
constexpr int kSmGroups = CSA_ATTN_GROUPS;      // softmax warpgroups (2 or 4)
constexpr int kSmWarps = 4 * kSmGroups;
constexpr int kHW = kNP / kSmGroups;            // heads per softmax warpgroup
// registers per thread after setmaxnreg: softmax / the rest.  The block is
// launched with 65536 / kThreads (rounded down to 8) per thread, and the split
// must add up to no more than that: 2 groups: 256 x 184 + 256 x 72 = 512 x 128;
// 4 groups: 512 x 88 + 256 x 64 = 768 x 80.
constexpr int kSmRegs = kSmGroups == 2 ? 184 : 88;
constexpr int kOtherRegs = kSmGroups == 2 ? 72 : 64;
constexpr int kMmaWarp = kSmWarps, kProducerWarp = kSmWarps + 1;
constexpr int kProducerWarps = 7;
constexpr int kProducerThreads = kProducerWarps * 32;
// kv_full arrivals per tile: one cp.async completion per producer thread plus
// one release arrive per producer warp (after its row-validity words)
constexpr uint32_t kKvFullCount = kProducerThreads + kProducerWarps;
constexpr int kThreads = (kSmWarps + 1 + kProducerWarps) * 32;
constexpr float kRescale = 8.f;                 // log2 units
constexpr int kTmemCols = 256;                  // S^T x2 (64 each) + O^T (64)
constexpr uint32_t kIdescS = tc::idesc_bf16(128, kNP, false, false);
constexpr uint32_t kIdescPV = tc::idesc_bf16(128, kNP, true, true);

// smem descriptor for the MN-major 128-byte swizzled operands: 8-row atoms
// (1024 B) along K at SBO = 1024, 64-element blocks along M/N at LBO.
__device__ __forceinline__ uint64_t desc_mn(uint32_t saddr, uint32_t lbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3fffu);
  d |= (uint64_t)((lbo >> 4) & 0x3fffu) << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

struct TcAttnParams {
  AttnArgs a;
  int hgroups;
  int64_t items;
  double theta[kD / 2];   // rotary pair frequencies base^(-2j / rope_dims) (host-filled)
};

// Position of query i for the rotary prologue / epilogue.
__device__ __forceinline__ int64_t rope_position(const AttnArgs& a, int64_t i) {
  return a.rope_pos ? __ldg(a.rope_pos + i) : (a.q_pos ? __ldg(a.q_pos + i) : i);
}

// cos / sin of the rotation of pair j at position p (R_p, or R_{-p} with
// inverse): the angle is formed and reduced modulo 2 pi in double precision
// (positions reach 2^20 and more), then sincosf.
__device__ __forceinline__ void rope_cs(const TcAttnParams& p, int64_t pos, int j, bool inverse,
                                        float& c, float& s) {
  const double two_pi = 6.283185307179586476925, inv_two_pi = 0.159154943091895335769;
  double ang = (double)pos * p.theta[j];
  ang -= two_pi * floor(ang * inv_two_pi);
  if (inverse) ang = -ang;
  sincosf((float)ang, &s, &c);
}

// Row list of one (query, split): selected / eligible entries [v0, min(v1, n_sel)),
// then window rows [max(v0, n_sel), v1) (virtual indices).
struct ItemInfo {
  int64_t i;        // query
  int split, hg;
  int64_t pos;
  int32_t seq;
  int64_t n_sel, n_win, win_first;
  int64_t v0, v1;
  int n_sel_tiles, n_tiles;
};

__device__ __forceinline__ ItemInfo item_info(const AttnArgs& a, int hgroups, int64_t item,
                                              bool do_report) {
  ItemInfo it;
  it.hg = (int)(item % hgroups);
  const int64_t rest = item / hgroups;
  it.split = (int)(rest % a.n_split);
  it.i = rest / a.n_split;
  it.pos = a.q_pos ? __ldg(a.q_pos + it.i) : it.i;
  it.seq = attn_seq(a, it.i);
  if (a.idx) {
    int64_t c = __ldg(a.count + it.i);
    it.n_sel = c < 0 ? 0 : (c > a.top_k ? a.top_k : c);
  } else {
    it.n_sel = it.pos / a.m;
    if (it.n_sel > a.max_entries) {
      if (do_report && it.split == 0 && it.hg == 0) report(a.err, kErrEligible, (int32_t)it.i, it.n_sel);
      it.n_sel = a.max_entries;
    }
  }
  it.win_first = 0;
  if (a.win_len) {
    it.n_win = __ldg(a.win_len + it.i);
    if (it.n_win < 0 || it.n_win > a.window) {
      if (do_report && it.split == 0 && it.hg == 0) report(a.err, kErrWindow, (int32_t)it.i, it.n_win);
      it.n_win = it.n_win < 0 ? 0 : a.window;
    }
  } else {
    it.win_first = attn_raw_window(a, it.i, it.pos, it.n_win, do_report && it.split == 0 && it.hg == 0);
  }
  const int64_t total = it.n_sel + it.n_win;
  it.v0 = (int64_t)it.split * a.split_len;
  it.v1 = total < it.v0 + a.split_len ? total : it.v0 + a.split_len;
  if (it.v1 < it.v0) it.v1 = it.v0;
  const int64_t s_end = it.v1 < it.n_sel ? it.v1 : it.n_sel;
  const int64_t w_beg = it.v0 > it.n_sel ? it.v0 : it.n_sel;
  it.n_sel_tiles = s_end > it.v0 ? (int)((s_end - it.v0 + kRows - 1) / kRows) : 0;
  const int n_win_tiles = it.v1 > w_beg ? (int)((it.v1 - w_beg + kRows - 1) / kRows) : 0;
  it.n_tiles = it.n_sel_tiles + n_win_tiles;
  return it;
}

// Tile t of an item: first virtual row and number of rows.
__device__ __forceinline__ void tile_span(const ItemInfo& it, int t, int64_t& v, int& n) {
  if (t < it.n_sel_tiles) {
    v = it.v0 + (int64_t)t * kRows;
    const int64_t e = it.v1 < it.n_sel ? it.v1 : it.n_sel;
    n = (int)(e - v < kRows ? e - v : kRows);
  } else {
    const int64_t w_beg = it.v0 > it.n_sel ? it.v0 : it.n_sel;
    v = w_beg + (int64_t)(t - it.n_sel_tiles) * kRows;
    n = (int)(it.v1 - v < kRows ? it.v1 - v : kRows);
  }
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

// a * b + c and a + b on two fp32 lanes per instruction (fma.rn / add.rn
// .f32x2: each lane rounds as fmaf / fadd do)
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n .reg .b64 ra, rb, rc, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n mov.b64 rc, {%6, %7};\n"
      " fma.rn.f32x2 rd, ra, rb, rc;\n mov.b64 {%0, %1}, rd;\n}\n"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 d;
  asm("{\n .reg .b64 ra, rb, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
      " add.rn.f32x2 rd, ra, rb;\n mov.b64 {%0, %1}, rd;\n}\n"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

__device__ __forceinline__ float redux_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;\n" : "=f"(r) : "f"(v));
  return r;
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16};\n" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

// Softmax-warp group barrier on an mbarrier (count 4): bounded, so that a
// warp that gave up elsewhere cannot strand the others.
__device__ __forceinline__ bool group_sync(uint32_t bar, uint32_t& phase, int lane, long long limit) {
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
  const bool ok = mbar_wait(bar, phase, limit);
  phase ^= 1u;
  return ok;
}

// Producer gather of mixed-precision entries (kept out of line: its registers
// stay off the bf16 path).  Lane (c = lane & 15, sub = lane >> 4) handles
// chunk c of row 2 (pk + kProducerWarps j) + sub of each of the warp's pairs
// j; `row` is lane l's physical row for pair l >> 1 (or -1).  Chunk c < dc8
// is 8 E4M3 codes and the scale byte of their block, expanded exactly to bf16
// and stored in the chunk's swizzled place (zeros for a missing row, as the
// zero fill of a bf16 row); the rotary chunks arrive by cp.async.  A few rows
// at a time: their loads are all issued before the first expansion.
__device__ __noinline__ void gather_fp8_rows(const uint8_t* codes, const uint8_t* scales,
                                             const __nv_bfloat16* rope, int rope_dims, uint32_t cdst,
                                             int64_t row, int my_pairs, int pk, int lane) {
  constexpr int kJ = (kRows / 2 + kProducerWarps - 1) / kProducerWarps;
  constexpr int kFB = kJ;   // all of the warp's rows in one batch: one round trip per tile
  const int c = lane & 15, sub = lane >> 4;
  const int dc8 = (kD - rope_dims) / 8;
#pragma unroll
  for (int j0 = 0; j0 < kJ; j0 += kFB) {
    uint2 cw[kFB];
    uint32_t sbyte[kFB];
#pragma unroll
    for (int u = 0; u < kFB; ++u) {
      const int j = j0 + u;
      cw[u] = make_uint2(0u, 0u);
      sbyte[u] = 0u;
      const int64_t rr = __shfl_sync(0xffffffffu, row, (2 * j + sub) & 31);
      if (j < kJ && j < my_pairs) {
        const int r = 2 * (pk + kProducerWarps * j) + sub;
        if (c < dc8) {
          if (rr >= 0) {
            cw[u] = __ldg(reinterpret_cast<const uint2*>(codes + rr * (8 * dc8) + 8 * c));
            sbyte[u] = __ldg(scales + rr * (dc8 / 4) + (c >> 2));
          }
        } else {
          cp_async_16(cdst + (uint32_t)r * 128 + (uint32_t)((((c & 7) ^ (r & 7)) & 7) << 4),
                      rope + (rr >= 0 ? rr : 0) * rope_dims + (c - dc8) * 8, rr >= 0);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kFB; ++u) {
      const int j = j0 + u;
      if (j < kJ && j < my_pairs && c < dc8) {
        const int r = 2 * (pk + kProducerWarps * j) + sub;
        const float fs = lowprec::e8m0_to_float(sbyte[u]);
        const uint32_t w2[2] = {cw[u].x, cw[u].y};
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) o[q] = lowprec::e4m3x2_scaled_bf16x2(w2[q >> 1] >> (16 * (q & 1)), fs);
        const uint32_t addr = cdst + (uint32_t)r * 128 + (uint32_t)((((c & 7) ^ (r & 7)) & 7) << 4);
        asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(addr), "r"(o[0]), "r"(o[1]),
                     "r"(o[2]), "r"(o[3])
                     : "memory");
      }
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_kv_tile,
               const __grid_constant__ CUtensorMap tm_win,
               const __grid_constant__ CUtensorMap tm_q, TcAttnParams p) {
  pdl_trigger();
  const AttnArgs& a = p.a;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t kv_full[kStages], kv_empty[kStages];
  __shared__ __align__(8) uint64_t q_full[2], q_empty[2], s_full[2], s_empty[2], p_full[2], p_empty[2];
  __shared__ __align__(8) uint64_t o_full, o_empty, o_step, red_bar[kSmGroups];
  // query prologue: the tile is normalised / rotated in place before S^T
  __shared__ __align__(8) uint64_t q_ready[2], pro_bar;
  __shared__ float2 rope_tab[2][kD / 2];   // cos / sin per pair, by Q buffer
  __shared__ uint32_t tmem_base_sh;
  // validity of the tile's rows, one word per producer warp: bit 2j + s of
  // word k is row 2 (k + 7 j) + s
  __shared__ uint32_t row_ok[kStages][8];
  __shared__ __align__(16) float red_max[2][kSmWarps][kHW];   // per-warp tile maxima, by tile parity
  __shared__ float red_l[kSmWarps][kHW];        // per-warp row sums at the end of an item
  __shared__ __align__(16) float w_bcast[kSmWarps][2 * kHW];   // per warp: exponent offsets, factors

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t q_sm = base;                                 // 2 x 16 KB
  const uint32_t kv_sm = base + 2 * kQTile;                   // kStages x 32 KB
  const uint32_t p_sm = kv_sm + kStages * kKvTile;            // 2 x 16 KB

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&kv_full[s]), kKvFullCount);
      mbar_init(smem_u32(&kv_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&q_full[s]), 1);
      mbar_init(smem_u32(&q_empty[s]), 1);
      mbar_init(smem_u32(&s_full[s]), 1);
      mbar_init(smem_u32(&s_empty[s]), kSmWarps);
      mbar_init(smem_u32(&p_full[s]), kSmWarps);
      mbar_init(smem_u32(&p_empty[s]), 1);
    }
    mbar_init(smem_u32(&o_full), 1);
    mbar_init(smem_u32(&o_empty), kSmWarps);
    mbar_init(smem_u32(&o_step), 1);
    mbar_init(smem_u32(&q_ready[0]), kSmWarps);
    mbar_init(smem_u32(&q_ready[1]), kSmWarps);
    mbar_init(smem_u32(&pro_bar), kSmWarps);
    for (int g = 0; g < kSmGroups; ++g) mbar_init(smem_u32(&red_bar[g]), 4);
    mbar_fence_init();
  }
  if (warp == kMmaWarp) tc::tmem_alloc(smem_u32(&tmem_base_sh), kTmemCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  // everything above overlaps the previous kernel's tail; nothing below may
  // read its outputs (selected entries, counts) before it has completed
  pdl_wait();
  const uint32_t tmem_base = tmem_base_sh;
  const uint32_t tm_s = tmem_base;              // two 64-column S^T buffers
  const uint32_t tm_o = tmem_base + 2 * kNP;    // O^T
  const int64_t n_items = p.items;

  // Registers: the MMA and producer warpgroups give theirs down to 72 per
  // thread, the softmax warpgroups take 184 (2 x 128 x (72 + 184) = the
  // 512 x 128 the block is launched with).
  if (warp >= kMmaWarp) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kOtherRegs) : "memory");
  if (warp >= kProducerWarp) {
    // ================================================================ producer
    // Seven warps.  Gathered rows: the tile's 64 row pairs are dealt round
    // robin (pair p to warp p mod 7); lane l of a warp resolves the row
    // 2 (pk + 7 (l >> 1)) + (l & 1) and the warp copies its rows with 16-byte
    // cp.async, 16 lanes per 256-byte row, two rows per instruction.  Several
    // warps keep enough copies in flight to stream the gather.  Contiguous
    // rows: one thread issues two 128-row TMA boxes.
    const int pk = warp - kProducerWarp;              // 0 .. kProducerWarps - 1
    const int pt = threadIdx.x - kProducerWarp * 32;
    const int my_pairs = (kRows / 2 - pk + kProducerWarps - 1) / kProducerWarps;
    const bool lane_has_row = (lane >> 1) < my_pairs;
    const int my_row = 2 * (pk + kProducerWarps * (lane >> 1)) + (lane & 1);
    if (pt == 0) {
      tc::prefetch_tmap(&tm_kv_tile);
      tc::prefetch_tmap(&tm_win);
      tc::prefetch_tmap(&tm_q);
    }
    int64_t tiles_done = 0, items_done = 0;
    bool ok = true;
    for (int64_t item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
      const ItemInfo it = item_info(a, p.hgroups, item, pt == 0);
      if (it.n_tiles == 0) continue;
      if (pt == 0) {   // the query's heads, once per item
        const int qb = (int)(items_done & 1);
        if (!mbar_wait(smem_u32(&q_empty[qb]), (uint32_t)(((items_done >> 1) & 1) ^ 1), a.wait_limit)) {
          report(a.err, kErrTimeout, (int32_t)it.i, 20);
          ok = false;
        } else if (!(a.withhold_q && items_done == 0)) {   // (test hook: never arrives)
          mbar_arrive_expect_tx(smem_u32(&q_full[qb]), kQTile);
          const int32_t qrow = (int32_t)(it.i * a.H + it.hg * kNP);
          const uint32_t qd = q_sm + qb * kQTile;
          tc::tma_load_2d(qd, &tm_q, 0, qrow, smem_u32(&q_full[qb]));
          tc::tma_load_2d(qd + kQTile / 2, &tm_q, 64, qrow, smem_u32(&q_full[qb]));
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);   // keep each warp's control flow uniform
      if (!ok) break;
      ++items_done;
      int64_t e_next = -1;   // this lane's entry id in the item's next gathered tile
      bool have_next = false;
      for (int t = 0; t < it.n_tiles && ok; ++t, ++tiles_done) {
        const int slot = (int)(tiles_done % kStages);
        const bool got =
            mbar_wait(smem_u32(&kv_empty[slot]), (uint32_t)(((tiles_done / kStages) & 1) ^ 1), a.wait_limit);
        if (!__all_sync(0xffffffffu, got)) {
          if (pt == 0) report(a.err, kErrTimeout, (int32_t)it.i, 21);
          ok = false;
          break;
        }
        int64_t v;
        int n;
        tile_span(it, t, v, n);
        const uint32_t dst = kv_sm + slot * kKvTile;
        const uint32_t fb = smem_u32(&kv_full[slot]);
        const bool sel = t < it.n_sel_tiles;
        if (sel && (a.idx != nullptr || a.kv.page_table != nullptr || a.kv_fp8)) {
          const bool mine = lane_has_row && my_row < n;
          const int64_t e = have_next ? e_next
                                      : (!mine ? -1 : (a.idx ? (int64_t)__ldg(a.idx + it.i * a.top_k + v + my_row)
                                                             : v + my_row));
          // the next gathered tile's entry id loads while this tile is copied
          have_next = t + 1 < it.n_sel_tiles;
          if (have_next) {
            int64_t v2;
            int n2;
            tile_span(it, t + 1, v2, n2);
            const bool mine2 = lane_has_row && my_row < n2;
            e_next = !mine2 ? -1 : (a.idx ? (int64_t)__ldg(a.idx + it.i * a.top_k + v2 + my_row) : v2 + my_row);
          }
          const int64_t row = mine ? cache_row(a.kv, it.seq, e, a.err, (int32_t)it.i) : -1;
          const uint32_t okb = __ballot_sync(0xffffffffu, row >= 0);   // bit l: lane l's row
          if (lane == 0) row_ok[slot][pk] = okb;
          const int c = lane & 15, sub = lane >> 4;
          const uint32_t cdst = dst + (c >> 3) * kKBlock;
          constexpr int kJ = (kRows / 2 + kProducerWarps - 1) / kProducerWarps;
          if (!a.kv_fp8) {
#pragma unroll
            for (int j = 0; j < kJ; ++j) {
              if (j < my_pairs) {
                const int64_t rr = __shfl_sync(0xffffffffu, row, 2 * j + sub);
                const int r = 2 * (pk + kProducerWarps * j) + sub;
                const char* src = reinterpret_cast<const char*>(a.kv.data + (rr >= 0 ? rr : 0) * kD) + c * 16;
                cp_async_16(cdst + (uint32_t)r * 128 + (uint32_t)((((c & 7) ^ (r & 7)) & 7) << 4), src,
                            rr >= 0);
              }
            }
          } else {
            gather_fp8_rows(reinterpret_cast<const uint8_t*>(a.kv.data), a.kv_scales, a.kv_rope,
                            a.rope_dims, cdst, row, my_pairs, pk, lane);
            fence_async_smem();   // the MMAs read the expanded rows through the async proxy
          }
          cp_async_mbar_arrive_noinc(fb);
          __syncwarp();
          if (lane == 0) mbar_arrive(fb);   // releases this warp's row_ok word
        } else if (pk == 0) {
          // contiguous rows: eligible entries of a contiguous cache, or the window
          int64_t row0;
          const CUtensorMap* map;
          if (sel) {
            row0 = (int64_t)it.seq * a.kv.seq_stride + v;
            map = &tm_kv_tile;
            // rows past this sequence's stride or past the cache are masked
            int64_t lim = a.kv.n_rows - row0;
            if (a.kv.seq_stride > 0 && a.kv.seq_stride - v < lim) lim = a.kv.seq_stride - v;
            if (lim < n) {
              if (lane == 0) report(a.err, kErrEntryIndex, (int32_t)it.i, v + (lim > 0 ? lim : 0));
              n = lim > 0 ? (int)lim : 0;
            }
          } else {
            const int64_t w = v - it.n_sel;
            row0 = a.win_len ? it.i * a.window + w : it.win_first + w;
            map = &tm_win;
          }
          if (lane < kProducerWarps) {   // the validity word of producer warp `lane`
            uint32_t word = 0;
            for (int j = 0; lane + kProducerWarps * j < kRows / 2; ++j) {
              const int r = 2 * (lane + kProducerWarps * j);
              if (r < n) word |= 1u << (2 * j);
              if (r + 1 < n) word |= 2u << (2 * j);
            }
            row_ok[slot][lane] = word;
            if (lane > 0) mbar_arrive(fb);   // releases its word
          }
          if (lane == 0) {
            mbar_expect_tx(fb, kKvTile);
            tc::tma_load_2d(dst, map, 0, (int32_t)row0, fb);
            tc::tma_load_2d(dst + kKBlock, map, 64, (int32_t)row0, fb);
            mbar_arrive_cnt(fb, kKvFullCount - (kProducerWarps - 1));
          }
        }
      }
    }
    // no copy of this thread may still be landing when the CTA exits
    cp_async_commit();
    cp_async_wait<0>();
    if (!ok && pt == 0) {
      const int64_t first = tiles_done > kStages ? tiles_done - kStages : 0;
      for (int64_t d = first; d < tiles_done; ++d)
        mbar_wait(smem_u32(&kv_full[d % kStages]), (uint32_t)((d / kStages) & 1), 200000000ll);
      if (items_done > 0 && !(a.withhold_q && items_done == 1))   // no query copy was issued
        mbar_wait(smem_u32(&q_full[(items_done - 1) & 1]), (uint32_t)(((items_done - 1) >> 1) & 1),
                  200000000ll);
    }
  } else {
    // ================================================================ MMA
    if (lane == 0) {
      int64_t tiles_done = 0, items_done = 0, pv_done = 0;
      bool ok = true;
      auto do_pv = [&](int64_t gtile, bool first) -> bool {
        const int pb = (int)(gtile & 1);
        if (!mbar_wait(smem_u32(&p_full[pb]), (uint32_t)((gtile >> 1) & 1), a.wait_limit)) return false;
        // the previous item's epilogue must have read O^T before it is overwritten
        if (first && !mbar_wait(smem_u32(&o_empty), (uint32_t)((items_done & 1) ^ 1), a.wait_limit)) return false;
        tc::fence_after_sync();
        const uint32_t kv = kv_sm + (int)(gtile % kStages) * kKvTile;
        const uint32_t pt = p_sm + pb * kPTile;
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk)
          tc::mma_bf16_ss(tm_o, desc_mn(kv + kk * 2048, kKBlock), desc_mn(pt + kk * 2048, kPTile),
                          kIdescPV, !(first && kk == 0));
        tc::mma_commit(smem_u32(&kv_empty[gtile % kStages]));
        tc::mma_commit(smem_u32(&p_empty[pb]));
        tc::mma_commit(smem_u32(&o_step));
        ++pv_done;
        return true;
      };
      for (int64_t item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        const ItemInfo it = item_info(a, p.hgroups, item, false);
        if (it.n_tiles == 0) continue;
        const int qb = (int)(items_done & 1);
        const uint32_t qs = q_sm + qb * kQTile;
        if (!mbar_wait(smem_u32(a.qprologue ? &q_ready[qb] : &q_full[qb]), (uint32_t)((items_done >> 1) & 1), a.wait_limit)) {
          report(a.err, kErrTimeout, (int32_t)it.i, 22);
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const int64_t first_tile = tiles_done;
        for (int t = 0; t < it.n_tiles; ++t, ++tiles_done) {
          const int slot = (int)(tiles_done % kStages);
          const int sb = (int)(tiles_done & 1);
          if (!mbar_wait(smem_u32(&kv_full[slot]), (uint32_t)((tiles_done / kStages) & 1), a.wait_limit) ||
              !mbar_wait(smem_u32(&s_empty[sb]), (uint32_t)(((tiles_done >> 1) & 1) ^ 1), a.wait_limit)) {
            report(a.err, kErrTimeout, (int32_t)it.i, 23);
            ok = false;
            break;
          }
          tc::fence_after_sync();
          const uint32_t kv = kv_sm + slot * kKvTile;
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kKBlock + (kk & 3) * 32;
            const uint32_t qoff = (kk >> 2) * (kQTile / 2) + (kk & 3) * 32;
            tc::mma_bf16_ss(tm_s + sb * kNP, tc::smem_desc_sw128(kv + off),
                            tc::smem_desc_sw128(qs + qoff), kIdescS, kk > 0);
          }
          tc::mma_commit(smem_u32(&s_full[sb]));
          if (t == it.n_tiles - 1) tc::mma_commit(smem_u32(&q_empty[qb]));
          if (t > 0 && !do_pv(tiles_done - 1, tiles_done - 1 == first_tile)) {
            report(a.err, kErrTimeout, (int32_t)it.i, 24);
            ok = false;
            break;
          }
        }
        if (!ok) break;
        if (!do_pv(tiles_done - 1, tiles_done - 1 == first_tile)) {
          report(a.err, kErrTimeout, (int32_t)it.i, 25);
          ok = false;
          break;
        }
        tc::mma_commit(smem_u32(&o_full));
        ++items_done;
      }
    }
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kSmRegs) : "memory");
    // ================================================================ softmax + epilogue
    // Warpgroup wg (warps 4wg .. 4wg+3) owns heads [32 wg, 32 wg + 32) of every
    // tile: thread = row of S^T in the tile loop, = dim of O^T in the epilogue.
    // The four warps exchange only their per-head tile maxima; each warp then
    // derives the same running maxima itself (lane h holds head 32 wg + h).
    const int wg = warp >> 2, wq = warp & 3;
    const int hoff = wg * kHW;
    const int hl = lane & (kHW - 1);
    const int row = wq * 32 + lane;
    const int ok_word = (row >> 1) % kProducerWarps, ok_bit = 2 * ((row >> 1) / kProducerWarps) + (row & 1);
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    const uint32_t rbar = smem_u32(&red_bar[wg]);
    const float scale = a.sm_scale * kLog2e;
    float* const my_bc = w_bcast[warp];   // this warp's per-head broadcast row
    uint32_t red_phase = 0, pro_phase = 0;
    int64_t tiles_done = 0, items_done = 0, pv_seen = 0;
    for (int64_t item = blockIdx.x; item < n_items; item += gridDim.x) {
      const ItemInfo it = item_info(a, p.hgroups, item, false);
      const int h_base = it.hg * kNP;
      const int nh = a.H - h_base < kNP ? a.H - h_base : kNP;
      if (it.n_tiles == 0) {
        // no rows: an empty partial for the merge, or a zero output
        for (int hl = 0; hl < kHW; ++hl) {
          const int h = hoff + hl;
          if (h >= nh) break;
          const int hh = h_base + h;
          if (a.n_split == 1) {
            a.out[(it.i * a.H + hh) * kD + row] = __float2bfloat16_rn(0.f);
            if (a.lse && row == 0) a.lse[it.i * a.H + hh] = a.sink ? __ldg(a.sink + hh) : -INFINITY;
          } else {
            const int64_t pb = (it.i * a.n_split + it.split) * a.H + hh;
            a.part_acc[pb * kD + row] = 0.f;
            if (row == 0) *reinterpret_cast<float2*>(a.part_ml + pb * 2) = make_float2(-INFINITY, 0.f);
          }
        }
        continue;
      }
      if (a.qprologue) {
        // ---------------------------------------------------- query prologue
        // RMSNorm (times the gain) and the rotation R_t of every head of this
        // item's query tile, in place in shared memory: thread = (head,
        // quarter of the dims), four 16-byte chunks of the swizzled tile.
        const int qb = (int)(items_done & 1);
        bool okp = mbar_wait(smem_u32(&q_full[qb]), (uint32_t)((items_done >> 1) & 1), a.wait_limit);
        const int r0 = kD - a.q_rope_dims;
        if (okp && a.q_rope_dims > 0 && (int)threadIdx.x < a.q_rope_dims / 2) {
          float c, sn;
          rope_cs(p, rope_position(a, it.i), threadIdx.x, false, c, sn);
          rope_tab[qb][threadIdx.x] = make_float2(c, sn);
        }
        okp = okp && group_sync(smem_u32(&pro_bar), pro_phase, lane, a.wait_limit);
        if (!okp) {
          if (lane == 0) report(a.err, kErrTimeout, (int32_t)it.i, 30);
          break;
        }
        const int head = threadIdx.x >> 2, qq = threadIdx.x & 3;
        uint8_t* const qtile = smem_raw + (q_sm + qb * kQTile - smem_u32(smem_raw));
        float x[32];
#pragma unroll
        for (int i = 0; i < 4; ++i) {   // chunk cc = dims [8 cc, 8 cc + 8)
          const int cc = 4 * qq + i, blk = cc >> 3, cb = cc & 7;
          const uint4 v = *reinterpret_cast<const uint4*>(qtile + blk * (kQTile / 2) + head * 128 +
                                                          ((cb ^ (head & 7)) << 4));
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f2 = unpack_bf16(w4[e]);
            x[8 * i + 2 * e] = f2.x;
            x[8 * i + 2 * e + 1] = f2.y;
          }
        }
        if (a.q_norm_eps >= 0.f) {
          float ss = 0.f;
#pragma unroll
          for (int e = 0; e < 32; ++e) ss = fmaf(x[e], x[e], ss);
          ss += __shfl_xor_sync(0xffffffffu, ss, 1);
          ss += __shfl_xor_sync(0xffffffffu, ss, 2);
          const float rn = fminf(rsqrtf(ss / (float)kD + a.q_norm_eps), 3.0e38f);   // zero rows stay zero
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float gv = a.q_norm_gain ? __ldg(a.q_norm_gain + 32 * qq + e) : 1.f;
            x[e] *= rn * gv;
          }
        }
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int dim = 32 * qq + e;
          if (a.q_rope_dims > 0 && dim >= r0) {
            const float2 cs = rope_tab[qb][(dim - r0) >> 1];
            const float u = x[e], w = x[e + 1];
            x[e] = u * cs.x - w * cs.y;
            x[e + 1] = u * cs.y + w * cs.x;
          }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int cc = 4 * qq + i, blk = cc >> 3, cb = cc & 7;
          uint4 v;
          v.x = pack_bf16(x[8 * i], x[8 * i + 1]);
          v.y = pack_bf16(x[8 * i + 2], x[8 * i + 3]);
          v.z = pack_bf16(x[8 * i + 4], x[8 * i + 5]);
          v.w = pack_bf16(x[8 * i + 6], x[8 * i + 7]);
          *reinterpret_cast<uint4*>(qtile + blk * (kQTile / 2) + head * 128 + ((cb ^ (head & 7)) << 4)) = v;
        }
        fence_async_smem();   // the MMA reads the tile through the async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&q_ready[qb]));
      }
      float m_run = -INFINITY;   // lane h: running max of head hoff + h, log2 units
      float lpart[kHW];
#pragma unroll
      for (int h = 0; h < kHW; ++h) lpart[h] = 0.f;
      bool ok = true;
      for (int t = 0; t < it.n_tiles && ok; ++t, ++tiles_done) {
        const int slot = (int)(tiles_done % kStages);
        const int sb = (int)(tiles_done & 1);
        ok = mbar_wait(smem_u32(&s_full[sb]), (uint32_t)((tiles_done >> 1) & 1), a.wait_limit) &&
             mbar_wait(smem_u32(&kv_full[slot]), (uint32_t)((tiles_done / kStages) & 1), a.wait_limit);
        if (!ok) break;
        tc::fence_after_sync();
        float x[kHW];
        {
          uint32_t rr[kHW / 16][16];
#pragma unroll
          for (int c = 0; c < kHW / 16; ++c) tc::tmem_ld16(tm_s + sb * kNP + hoff + 16 * c + lane_base, rr[c]);
          tc::tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < kHW / 16; ++c)
#pragma unroll
            for (int j = 0; j < 16; ++j) x[16 * c + j] = __uint_as_float(rr[c][j]);
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&s_empty[sb]));
        const bool valid = (row_ok[slot][ok_word] >> ok_bit) & 1u;
        if (!__all_sync(0xffffffffu, valid)) {   // rows past the list or without an entry
#pragma unroll
          for (int h = 0; h < kHW; ++h)
            if (!valid) x[h] = -INFINITY;
        }
        // per-head tile maxima of the raw logits across this warp's 32 rows
        // (warp-uniform after the reduction; lane 0 publishes them)
        float (*const rm)[kHW] = red_max[sb];
        {
          float mx[kHW];
#pragma unroll
          for (int h = 0; h < kHW; ++h) mx[h] = redux_max(x[h]);
          if (lane == 0) {
#pragma unroll
            for (int h = 0; h < kHW; h += 4)
              *reinterpret_cast<float4*>(&rm[warp][h]) = make_float4(mx[h], mx[h + 1], mx[h + 2], mx[h + 3]);
          }
        }
        if (!(ok = group_sync(rbar, red_phase, lane, a.wait_limit))) break;
        // lane hl = lane mod kHW stands for head hoff + hl (lanes past kHW repeat them)
        float tmax = fmaxf(fmaxf(rm[4 * wg][hl], rm[4 * wg + 1][hl]),
                           fmaxf(rm[4 * wg + 2][hl], rm[4 * wg + 3][hl]));
        tmax *= scale;   // scale > 0: the max commutes with it
        float f = 1.f;
        bool grew = false;
        if (tmax > m_run + kRescale || (m_run == -INFINITY && tmax > -INFINITY)) {
          f = m_run == -INFINITY ? 0.f : exp2f(m_run - tmax);
          grew = m_run != -INFINITY;
          m_run = tmax;
        }
        const bool rescale = __any_sync(0xffffffffu, grew);
        if (lane < kHW) {
          my_bc[lane] = m_run == -INFINITY ? 0.f : -m_run;   // negated: the exponent is s scale + this
          if (rescale) my_bc[kHW + lane] = f;
        }
        __syncwarp();
        if (rescale) {
          // this warp's 32 dims of O^T for the group's heads, when a running max moved
          if (pv_seen < tiles_done) {   // every earlier PV must have completed
            if (!(ok = mbar_wait(smem_u32(&o_step), (uint32_t)((tiles_done - 1) & 1), a.wait_limit))) break;
            pv_seen = tiles_done;
          }
          tc::fence_after_sync();
#pragma unroll
          for (int c = 0; c < kHW / 16; ++c) {
            uint32_t r[16];
            tc::tmem_ld16(tm_o + hoff + c * 16 + lane_base, r);
            tc::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j)
              r[j] = __float_as_uint(__uint_as_float(r[j]) * my_bc[kHW + c * 16 + j]);
            tmem_st16(tm_o + hoff + c * 16 + lane_base, r);
          }
          tmem_wait_st();
          tc::fence_before_sync();
        }
        // probabilities, partial sums, bf16 P^T (this group's 64 bytes of the row)
        if (!(ok = mbar_wait(smem_u32(&p_empty[sb]), (uint32_t)(((tiles_done >> 1) & 1) ^ 1), a.wait_limit))) break;
        const uint32_t prow = p_sm + sb * kPTile + (uint32_t)row * 128;
#pragma unroll
        for (int c = 0; c < kHW / 8; ++c) {
          const float4 me0 = *reinterpret_cast<const float4*>(my_bc + c * 8);
          const float4 me1 = *reinterpret_cast<const float4*>(my_bc + c * 8 + 4);
          const float nme[8] = {me0.x, me0.y, me0.z, me0.w, me1.x, me1.y, me1.z, me1.w};
          uint32_t pk[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int hl = c * 8 + 2 * j;
            // two heads per instruction: exponent, then the running row sums
            const float2 e2 = fma2(make_float2(x[hl], x[hl + 1]), make_float2(scale, scale),
                                   make_float2(nme[2 * j], nme[2 * j + 1]));
            const float2 p = make_float2(ex2_approx(e2.x), ex2_approx(e2.y));
            const float2 lp = rescale ? fma2(make_float2(lpart[hl], lpart[hl + 1]),
                                             make_float2(my_bc[kHW + hl], my_bc[kHW + hl + 1]), p)
                                      : add2(make_float2(lpart[hl], lpart[hl + 1]), p);
            lpart[hl] = lp.x;
            lpart[hl + 1] = lp.y;
            pk[j] = pack_bf16(p.x, p.y);
          }
          const int chunk = hoff / 8 + c;
          const uint32_t dst = prow + (uint32_t)(((chunk ^ (row & 7)) & 7) << 4);
          asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(dst), "r"(pk[0]), "r"(pk[1]),
                       "r"(pk[2]), "r"(pk[3])
                       : "memory");
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&p_full[sb]));
      }
      if (!ok) {
        if (lane == 0) report(a.err, kErrTimeout, (int32_t)it.i, 26);
        break;
      }
      // ------------------------------------------------------------ epilogue
      // Compact on purpose: it runs once per item, so it is cold in the
      // instruction cache; rolled loops keep it short.
      // Row sums: a butterfly leaves lane h with this warp's sum for head h,
      // the four warps' sums meet in shared memory.
#pragma unroll
      for (int sh = kHW / 2; sh >= 1; sh >>= 1) {
        const bool upper = (lane & sh) != 0;
#pragma unroll
        for (int j = 0; j < sh; ++j) {
          const float send = upper ? lpart[j] : lpart[j + sh];
          const float keep = upper ? lpart[j + sh] : lpart[j];
          lpart[j] = keep + __shfl_xor_sync(0xffffffffu, send, sh);
        }
      }
      for (int o = kHW; o < 32; o <<= 1) lpart[0] += __shfl_xor_sync(0xffffffffu, lpart[0], o);
      if (lane < kHW) red_l[warp][lane] = lpart[0];
      if (!mbar_wait(smem_u32(&o_full), (uint32_t)(items_done & 1), a.wait_limit) ||
          !group_sync(rbar, red_phase, lane, a.wait_limit)) {
        if (lane == 0) report(a.err, kErrTimeout, (int32_t)it.i, 28);
        break;
      }
      pv_seen = tiles_done;
      {
        const int h = hoff + hl;
        const float l = (red_l[4 * wg][hl] + red_l[4 * wg + 1][hl]) +
                        (red_l[4 * wg + 2][hl] + red_l[4 * wg + 3][hl]);
        const float m = m_run;
        float nrm = 1.f;
        if (a.n_split == 1) {
          // normaliser (with the sink in the denominator) and log-sum-exp
          float den = l, f = 1.f, mm = m;
          if (a.sink != nullptr && h < nh) {
            const float z = __ldg(a.sink + h_base + h) * kLog2e;
            const float M = fmaxf(m, z);
            const float rr = M == -INFINITY ? 0.f : M;
            f = exp2f(m - rr);
            den = l * f + exp2f(z - rr);
            mm = rr;
          }
          nrm = den > 0.f ? __fdividef(f, den) : 0.f;
          if (wq == 0 && lane < kHW && a.lse != nullptr && h < nh)
            a.lse[it.i * a.H + h_base + h] = den > 0.f ? (mm + log2f(den)) / kLog2e : -INFINITY;
        } else if (wq == 0 && lane < kHW && h < nh) {
          *reinterpret_cast<float2*>(a.part_ml + ((it.i * a.n_split + it.split) * a.H + h_base + h) * 2) =
              make_float2(m, l);
        }
        if (lane < kHW) my_bc[kHW + lane] = nrm;
      }
      __syncwarp();
      tc::fence_after_sync();
      const int d = row;   // O^T lane = output dim
      // output de-rotation R_{-t} of the rotary pairs (2j, 2j+1): the pair's
      // two dims sit in neighbouring lanes; applied before normalisation or to
      // the split partials alike (both are linear in O)
      const bool derot = a.out_derotate && d >= kD - a.q_rope_dims;
      float dc = 1.f, ds = 0.f;
      if (derot) rope_cs(p, rope_position(a, it.i), (d - (kD - a.q_rope_dims)) >> 1, true, dc, ds);
      const float dsig = (d & 1) ? ds : -ds;   // even: v c - partner s; odd: v c + partner s
      if (a.n_split == 1) {
        __nv_bfloat16* const outp = a.out + (it.i * a.H + h_base) * kD + d;
#pragma unroll 1
        for (int c = 0; c < kHW / 16; ++c) {
          uint32_t r[16];
          tc::tmem_ld16(tm_o + hoff + c * 16 + lane_base, r);
          tc::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int h = hoff + c * 16 + j;
            float v = __uint_as_float(r[j]) * my_bc[kHW + c * 16 + j];
            const float partner = __shfl_xor_sync(0xffffffffu, v, 1);
            if (derot) v = fmaf(v, dc, partner * dsig);
            if (h < nh) outp[(int64_t)h * kD] = __float2bfloat16_rn(v);
          }
        }
      } else {
        float* const accp = a.part_acc + ((it.i * a.n_split + it.split) * a.H + h_base) * kD + d;
#pragma unroll 1
        for (int c = 0; c < kHW / 16; ++c) {
          uint32_t r[16];
          tc::tmem_ld16(tm_o + hoff + c * 16 + lane_base, r);
          tc::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int h = hoff + c * 16 + j;
            float v = __uint_as_float(r[j]);
            const float partner = __shfl_xor_sync(0xffffffffu, v, 1);
            if (derot) v = fmaf(v, dc, partner * dsig);
            if (h < nh) accp[(int64_t)h * kD] = v;
          }
        }
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&o_empty));
      ++items_done;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == kMmaWarp) tc::tmem_dealloc(tmem_base, kTmemCols);
}

}  // namespace

bool tc_attention_supported(const AttnArgs& a) {
  if (a.d != kD) return false;
  if (a.T * (int64_t)a.H > INT32_MAX || a.kv.n_rows > INT32_MAX) return false;
  if (a.win_len == nullptr && a.window > 0 && a.win_rows <= 0) return false;   // raw rows unknown
  if (a.win_len && a.T * (int64_t)a.window > INT32_MAX) return false;
  return true;
}

cudaError_t launch_attention_tc(const Launch& L, const AttnArgs& a) {
  CUtensorMap t, w, q;
  const uint64_t kv_rows = (uint64_t)a.kv.n_rows;
  // (mixed-precision entries are always gathered: no tile of them is a box)
  if (!make_tmap_bf16_2d(&t, a.kv_fp8 ? (const void*)a.q : (const void*)a.kv.data, kD,
                         a.kv_fp8 ? (uint64_t)(a.T * a.H) : kv_rows, kD, 64, kRows))
    return cudaErrorInvalidValue;
  const uint64_t win_rows = a.win_len ? (uint64_t)(a.T * a.window) : (uint64_t)a.win_rows;
  if (a.window > 0 && win_rows > 0) {
    if (!make_tmap_bf16_2d(&w, a.win, kD, win_rows, kD, 64, kRows)) return cudaErrorInvalidValue;
  } else {
    w = t;   // no window rows are ever read
  }
  if (!make_tmap_bf16_2d(&q, a.q, kD, (uint64_t)(a.T * a.H), kD, 64, kNP)) return cudaErrorInvalidValue;
  TcAttnParams p;
  p.a = a;
  p.hgroups = (a.H + kNP - 1) / kNP;
  p.items = a.T * a.n_split * p.hgroups;
  for (int j = 0; j < kD / 2; ++j)
    p.theta[j] = j < a.q_rope_dims / 2
                     ? std::pow((double)a.q_rope_base, -2.0 * j / (double)a.q_rope_dims) : 0.0;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t grid = p.items < sms ? p.items : sms;
  if (grid < 1) return cudaSuccess;
  const int smem = 2 * kQTile + kStages * kKvTile + 2 * kPTile + 1024;
  cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  prefer_max_shared(attn_tc_kernel);
  return launch_kernel(attn_tc_kernel, dim3((unsigned)grid), dim3(kThreads), (size_t)smem, L.stream,
                       true, t, w, q, p);
}

}  // namespace csa
