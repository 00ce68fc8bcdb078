// Step 4: shared-KV softmax attention over gathered rows.
//
// DeepSeek-V4 book, Ch.6 "Shared key-value MQA" (every head reads the same
// vectors, each both key and value), Ch.7 "The 128-token uncompressed sliding
// window" (selected entries and window rows share one softmax), "Dense
// attention over heavily compressed history" (HCA: all s < floor(t/m)) and
// "Learned attention sinks" (exp(z'_h) joins the denominator).
//
// Each query has a virtual row list: its selected (CSA) or eligible (HCA)
// compressed entries, then its window rows.  A CTA takes one query, one slice
// of that list (split-KV) and up to 64 heads (16 per warp).  Rows are
// gathered 64 at a time with cp.async into a double-buffered, XOR-swizzled
// shared tile; QK^T and PV run on tensor cores (mma.sync m16n8k16, bf16 in,
// fp32 accumulate) with an online softmax in the log2 domain.  A slice writes
// either the final output (one slice) or (acc, max, sum) partials that the
// merge kernel combines.  With mixed-precision entries (E4M3 content with a
// scale byte per 32, bf16 rotary part: Ch.8 "V4 compressed-entry payload")
// the gather expands each entry exactly to bf16 in the tile, so the rest of
// the kernel is unchanged.
#include "kernels.h"
#include "lowprec.cuh"

namespace csa {

namespace {

constexpr int D = 128;

__device__ __forceinline__ uint32_t ld_u32(const __nv_bfloat16* p) {
  return *reinterpret_cast<const uint32_t*>(p);
}

// BN rows per tile (32 or 64): with few warps per CTA the 2 x BN x 256 B of
// row tiles is what limits the CTAs resident on an SM.  One-warp CTAs are
// held to 168 registers so that 12 fit on an SM (L = 4096, H = 8, k = 64:
// 70.2 -> 68.0 us; 16 per SM, at 128 registers, spilled: 80.4 us).
template <int NW, int BN>
__global__ void __launch_bounds__(NW * 32, NW == 1 ? 12 : 1) attn_kernel(AttnArgs a) {
  static_assert(BN == 32 || BN == 64, "row tiles of 32 or 64");
  constexpr int NTH = NW * 32;
  __shared__ alignas(128) __nv_bfloat16 sKV[2][BN * D];
  __shared__ const __nv_bfloat16* sRow[2][BN];
  __shared__ int64_t sPhys[2][BN];   // mixed-precision entries: physical row, else -1
  __shared__ uint32_t sMask[2][2];

  const int64_t i = blockIdx.x;
  const int split = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, q4 = lane & 3;
  const int head0 = (blockIdx.z * NW + warp) * 16;

  // ---- this query's virtual row list ----
  const int64_t pos = a.q_pos ? __ldg(a.q_pos + i) : i;
  const int32_t seq = attn_seq(a, i);
  int64_t n_sel;
  if (a.idx) {
    n_sel = __ldg(a.count + i);
    n_sel = n_sel < 0 ? 0 : (n_sel > a.top_k ? a.top_k : n_sel);
  } else {
    n_sel = pos / a.m;
    if (n_sel > a.max_entries) {
      if (split == 0 && tid == 0 && blockIdx.z == 0) report(a.err, kErrEligible, (int32_t)i, n_sel);
      n_sel = a.max_entries;
    }
  }
  int64_t n_win, win_first = 0;
  if (a.win_len) {
    n_win = __ldg(a.win_len + i);
    if (n_win < 0 || n_win > a.window) {
      if (split == 0 && tid == 0 && blockIdx.z == 0) report(a.err, kErrWindow, (int32_t)i, n_win);
      n_win = n_win < 0 ? 0 : a.window;
    }
  } else {
    win_first = attn_raw_window(a, i, pos, n_win, split == 0 && tid == 0 && blockIdx.z == 0);
  }
  const int64_t total = n_sel + n_win;
  const int64_t v0 = (int64_t)split * a.split_len;
  const int64_t v1 = total < v0 + a.split_len ? total : v0 + a.split_len;
  const int ntiles = v1 > v0 ? (int)((v1 - v0 + BN - 1) / BN) : 0;

  // A row of the list is a bf16 row (sRow) or, with mixed-precision entries,
  // the physical row of an entry (sPhys); invalid rows have neither.
  auto fill_rows = [&](int st, int tt) {
    for (int r0 = warp * 32; r0 < BN; r0 += NTH) {
      const int r = r0 + lane;
      const int64_t v = v0 + (int64_t)tt * BN + r;
      const __nv_bfloat16* p = nullptr;
      int64_t phys = -1;
      if (v < v1) {
        if (v < n_sel) {
          const int64_t e = a.idx ? (int64_t)__ldg(a.idx + i * a.top_k + v) : v;
          const int64_t rr = cache_row(a.kv, seq, e, a.err, (int32_t)i);
          if (rr >= 0) {
            if (a.kv_fp8) phys = rr;
            else p = a.kv.data + rr * D;
          }
        } else {
          const int64_t w = v - n_sel;
          p = a.win_len ? a.win + (i * a.window + w) * D : a.win + (win_first + w) * D;
        }
      }
      sRow[st][r] = p;
      sPhys[st][r] = phys;
      const uint32_t bits = __ballot_sync(0xffffffffu, p != nullptr || phys >= 0);
      if (lane == 0) sMask[st][r0 >> 5] = bits;
    }
  };
  // bf16 rows (and the rotary part of mixed-precision entries) arrive by
  // cp.async; an entry's E4M3 content is loaded, scaled and stored as exact
  // bf16 values in the same swizzled place
  const int dc8 = (D - a.rope_dims) / 8;   // 16-byte chunks of E4M3 content
  const uint8_t* kv_codes = reinterpret_cast<const uint8_t*>(a.kv.data);
  auto issue_tile = [&](int st) {
    const uint32_t base = smem_u32(sKV[st]);
#pragma unroll
    for (int c = tid; c < BN * 16; c += NTH) {
      const int r = c >> 4, ch = c & 15;
      const __nv_bfloat16* src = sRow[st][r];
      const uint32_t off = (uint32_t)(r * D + ((ch ^ (r & 7)) << 3));
      const int64_t phys = a.kv_fp8 ? sPhys[st][r] : -1;
      if (phys < 0) {
        cp_async_16(base + off * 2u, src ? src + ch * 8 : a.q, src != nullptr);
      } else if (ch < dc8) {
        const uint2 cw = __ldg(reinterpret_cast<const uint2*>(kv_codes + phys * (8 * dc8) + 8 * ch));
        const float fs = lowprec::e8m0_to_float(__ldg(a.kv_scales + phys * (dc8 / 4) + (ch >> 2)));
        uint4 o;
        o.x = lowprec::e4m3x2_scaled_bf16x2(cw.x, fs);
        o.y = lowprec::e4m3x2_scaled_bf16x2(cw.x >> 16, fs);
        o.z = lowprec::e4m3x2_scaled_bf16x2(cw.y, fs);
        o.w = lowprec::e4m3x2_scaled_bf16x2(cw.y >> 16, fs);
        *reinterpret_cast<uint4*>(&sKV[st][off]) = o;
      } else {
        cp_async_16(base + off * 2u, a.kv_rope + phys * a.rope_dims + (ch - dc8) * 8, true);
      }
    }
  };

  // ---- query fragments (A operand, rows = heads) ----
  uint32_t qa[D / 16][4];
  {
    const int h_lo = head0 + g, h_hi = head0 + g + 8;
    const __nv_bfloat16* qlo = a.q + (i * a.H + h_lo) * D;
    const __nv_bfloat16* qhi = a.q + (i * a.H + h_hi) * D;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int c = kk * 16 + 2 * q4;
      qa[kk][0] = h_lo < a.H ? ld_u32(qlo + c) : 0u;
      qa[kk][1] = h_hi < a.H ? ld_u32(qhi + c) : 0u;
      qa[kk][2] = h_lo < a.H ? ld_u32(qlo + c + 8) : 0u;
      qa[kk][3] = h_hi < a.H ? ld_u32(qhi + c + 8) : 0u;
    }
  }
  const float scale = a.sm_scale * kLog2e;

  float acc[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;

  if (ntiles > 0) {
    fill_rows(0, 0);
    __syncthreads();
    issue_tile(0);
    cp_async_commit();
  }
  for (int tt = 0; tt < ntiles; ++tt) {
    const int st = tt & 1;
    if (tt + 1 < ntiles) fill_rows(st ^ 1, tt + 1);
    __syncthreads();
    if (tt + 1 < ntiles) issue_tile(st ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();

    const uint32_t sbase = smem_u32(sKV[st]);
    // S = Q K^T  (16 heads x 64 rows per warp)
    float s[BN / 8][4];
#pragma unroll
    for (int j = 0; j < BN / 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int jp = 0; jp < BN / 16; ++jp) {
        const int mi = lane >> 3, rr = lane & 7;
        const int row = 16 * jp + 8 * (mi >> 1) + rr;
        const int ch = 2 * kk + (mi & 1);
        uint32_t r[4];
        ldmatrix_x4(r, sbase + (uint32_t)(row * D + ((ch ^ (row & 7)) << 3)) * 2u);
        mma_bf16_16816(s[2 * jp], qa[kk], r[0], r[1]);
        mma_bf16_16816(s[2 * jp + 1], qa[kk], r[2], r[3]);
      }
    }
    // online softmax (log2 domain); rows g (lo) and g+8 (hi) of this warp
    const uint64_t vmask = (uint64_t)sMask[st][0] | ((uint64_t)sMask[st][1] << 32);
    float mx_lo = -INFINITY, mx_hi = -INFINITY;
#pragma unroll
    for (int j = 0; j < BN / 8; ++j) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const bool ok = (vmask >> (8 * j + 2 * q4 + c)) & 1ull;
        s[j][c] = ok ? s[j][c] * scale : -INFINITY;
        s[j][2 + c] = ok ? s[j][2 + c] * scale : -INFINITY;
        mx_lo = fmaxf(mx_lo, s[j][c]);
        mx_hi = fmaxf(mx_hi, s[j][2 + c]);
      }
    }
    mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 1));
    mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 2));
    mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 1));
    mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 2));
    const float mn_lo = fmaxf(m_lo, mx_lo), mn_hi = fmaxf(m_hi, mx_hi);
    const float ref_lo = mn_lo == -INFINITY ? 0.f : mn_lo;
    const float ref_hi = mn_hi == -INFINITY ? 0.f : mn_hi;
    const float al_lo = exp2f(m_lo - ref_lo), al_hi = exp2f(m_hi - ref_hi);
    m_lo = mn_lo;
    m_hi = mn_hi;
    l_lo *= al_lo;
    l_hi *= al_hi;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      acc[n][0] *= al_lo;
      acc[n][1] *= al_lo;
      acc[n][2] *= al_hi;
      acc[n][3] *= al_hi;
    }
    uint32_t pa[BN / 16][4];
#pragma unroll
    for (int j = 0; j < BN / 8; ++j) {
      const float p0 = exp2f(s[j][0] - ref_lo), p1 = exp2f(s[j][1] - ref_lo);
      const float p2 = exp2f(s[j][2] - ref_hi), p3 = exp2f(s[j][3] - ref_hi);
      l_lo += p0 + p1;
      l_hi += p2 + p3;
      pa[j >> 1][(j & 1) * 2 + 0] = pack_bf16(p0, p1);
      pa[j >> 1][(j & 1) * 2 + 1] = pack_bf16(p2, p3);
    }
    // O += P V
#pragma unroll
    for (int kk2 = 0; kk2 < BN / 16; ++kk2) {
#pragma unroll
      for (int np = 0; np < D / 16; ++np) {
        const int mi = lane >> 3, rr = lane & 7;
        const int row = 16 * kk2 + 8 * (mi & 1) + rr;
        const int ch = 2 * np + (mi >> 1);
        uint32_t r[4];
        ldmatrix_x4_trans(r, sbase + (uint32_t)(row * D + ((ch ^ (row & 7)) << 3)) * 2u);
        mma_bf16_16816(acc[2 * np], pa[kk2], r[0], r[1]);
        mma_bf16_16816(acc[2 * np + 1], pa[kk2], r[2], r[3]);
      }
    }
    __syncthreads();   // stage st and sRow[st] are refilled two tiles later
  }

  l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 1);
  l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 2);
  l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 1);
  l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 2);

  const int h_lo = head0 + g, h_hi = head0 + g + 8;
  if (a.n_split == 1) {
    float f_lo = 1.f, f_hi = 1.f, den_lo = l_lo, den_hi = l_hi;
    float mm_lo = m_lo, mm_hi = m_hi;
    if (a.sink) {
      const float z_lo = h_lo < a.H ? __ldg(a.sink + h_lo) * kLog2e : -INFINITY;
      const float z_hi = h_hi < a.H ? __ldg(a.sink + h_hi) * kLog2e : -INFINITY;
      const float M_lo = fmaxf(m_lo, z_lo), M_hi = fmaxf(m_hi, z_hi);
      const float r_lo = M_lo == -INFINITY ? 0.f : M_lo, r_hi = M_hi == -INFINITY ? 0.f : M_hi;
      f_lo = exp2f(m_lo - r_lo);
      f_hi = exp2f(m_hi - r_hi);
      den_lo = l_lo * f_lo + exp2f(z_lo - r_lo);
      den_hi = l_hi * f_hi + exp2f(z_hi - r_hi);
      mm_lo = r_lo;
      mm_hi = r_hi;
    }
    const float inv_lo = den_lo > 0.f ? f_lo / den_lo : 0.f;
    const float inv_hi = den_hi > 0.f ? f_hi / den_hi : 0.f;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      const int c = 8 * n + 2 * q4;
      if (h_lo < a.H)
        *reinterpret_cast<uint32_t*>(a.out + (i * a.H + h_lo) * D + c) =
            pack_bf16(acc[n][0] * inv_lo, acc[n][1] * inv_lo);
      if (h_hi < a.H)
        *reinterpret_cast<uint32_t*>(a.out + (i * a.H + h_hi) * D + c) =
            pack_bf16(acc[n][2] * inv_hi, acc[n][3] * inv_hi);
    }
    if (a.lse && q4 == 0) {
      if (h_lo < a.H) a.lse[i * a.H + h_lo] = den_lo > 0.f ? (mm_lo + log2f(den_lo)) / kLog2e : -INFINITY;
      if (h_hi < a.H) a.lse[i * a.H + h_hi] = den_hi > 0.f ? (mm_hi + log2f(den_hi)) / kLog2e : -INFINITY;
    }
  } else {
    const int64_t pbase = (i * a.n_split + split) * a.H;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
      const int c = 8 * n + 2 * q4;
      if (h_lo < a.H)
        *reinterpret_cast<float2*>(a.part_acc + (pbase + h_lo) * D + c) = make_float2(acc[n][0], acc[n][1]);
      if (h_hi < a.H)
        *reinterpret_cast<float2*>(a.part_acc + (pbase + h_hi) * D + c) = make_float2(acc[n][2], acc[n][3]);
    }
    if (q4 == 0) {
      if (h_lo < a.H) *reinterpret_cast<float2*>(a.part_ml + (pbase + h_lo) * 2) = make_float2(m_lo, l_lo);
      if (h_hi < a.H) *reinterpret_cast<float2*>(a.part_ml + (pbase + h_hi) * 2) = make_float2(m_hi, l_hi);
    }
  }
}

// Combine the split partials of one (query, head): 64 threads, 2 dims each.
// One warp per (query, head), 4 dims per lane.  Splits are taken in chunks
// of 16 whose loads are all issued before any is used (one memory round trip
// per chunk); the running maximum, denominator and output are rescaled between
// chunks.  The sink enters as one more term with logit z and no value.
constexpr int kMergeHeads = 4;   // warps per block
constexpr int kMergeChunk = 16;

__global__ void __launch_bounds__(32 * kMergeHeads) merge_kernel(AttnArgs a) {
  pdl_wait();   // the partials of the attention launch are complete
  pdl_trigger();
  const int64_t i = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y * kMergeHeads + warp;
  if (h >= a.H) return;
  const int ns = a.n_split;
  const int dd = a.d;   // 128 or 512: blocks of 128 dims, 4 per lane
  const float* const ml = a.part_ml + (i * ns * a.H + h) * 2;
  float M = 0.f, den = 0.f;   // the same for every block; the last one's is kept for the LSE
  for (int d0 = 0; d0 < dd; d0 += D) {
    const float* const acc = a.part_acc + (i * ns * a.H + h) * dd + d0 + 4 * lane;
    const float z = a.sink ? __ldg(a.sink + h) * kLog2e : -INFINITY;
    M = z;
    den = z == -INFINITY ? 0.f : 1.f;   // relative to 2^M
    float4 out = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < ns; s0 += kMergeChunk) {
      const int cnt = ns - s0 < kMergeChunk ? ns - s0 : kMergeChunk;
      float2 mls = make_float2(-INFINITY, 0.f);
      if (lane < cnt) mls = *reinterpret_cast<const float2*>(ml + (int64_t)(s0 + lane) * a.H * 2);
      float4 v[kMergeChunk];
#pragma unroll
      for (int j = 0; j < kMergeChunk; ++j)
        if (j < cnt) v[j] = *reinterpret_cast<const float4*>(acc + (int64_t)(s0 + j) * a.H * dd);
      float cm = mls.x;
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, o));
      const float nM = fmaxf(M, cm);
      const float ref = nM == -INFINITY ? 0.f : nM;
      const float fo = exp2f(M - ref);
      den *= fo;
      out.x *= fo;
      out.y *= fo;
      out.z *= fo;
      out.w *= fo;
      const float f_l = lane < cnt ? exp2f(mls.x - ref) : 0.f;
      float dl = f_l * mls.y;
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) dl += __shfl_xor_sync(0xffffffffu, dl, o);
      den += dl;
#pragma unroll
      for (int j = 0; j < kMergeChunk; ++j) {
        const float f = __shfl_sync(0xffffffffu, f_l, j);
        if (j < cnt) {
          out.x = fmaf(v[j].x, f, out.x);
          out.y = fmaf(v[j].y, f, out.y);
          out.z = fmaf(v[j].z, f, out.z);
          out.w = fmaf(v[j].w, f, out.w);
        }
      }
      M = nM;
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    uint2 pk;
    pk.x = pack_bf16(out.x * inv, out.y * inv);
    pk.y = pack_bf16(out.z * inv, out.w * inv);
    *reinterpret_cast<uint2*>(a.out + (i * a.H + h) * dd + d0 + 4 * lane) = pk;
  }
  const float ref = M == -INFINITY ? 0.f : M;
  if (a.lse && lane == 0) a.lse[i * a.H + h] = den > 0.f ? (ref + log2f(den)) / kLog2e : -INFINITY;
}

cudaError_t launch_merge(const Launch& L, const AttnArgs& a) {
  L.begin(kKernelMerge);
  const dim3 grid((unsigned)a.T, (unsigned)((a.H + kMergeHeads - 1) / kMergeHeads));
  prefer_max_shared(merge_kernel);
  const cudaError_t e = launch_kernel(merge_kernel, grid, dim3(32 * kMergeHeads), 0, L.stream, true, a);
  if (e != cudaSuccess) return e;
  return L.end(kKernelMerge);
}

}  // namespace

// The automatic choice.  Short row lists favour the mma.sync kernel: the
// tensor-core kernel's fixed cost per (query, slice) item (query tile, first
// scores, epilogue: about 4 us) then outweighs its tiles.  Measured at
// L = 4096, m = 4, W = 128 with H from 8 to 64: k = 64 (at most 192 rows)
// 72-150 us against 179-182 us.  So do few heads over many queries: the
// tensor-core kernel still runs 64-head tiles, while the mma.sync kernel
// takes one warp (and 32-row tiles) per 16 heads: with H = 8 or 16, k = 512
// to 2048 and 4096 to 16384 queries, 195-1837 us against 252-2338 us.  With
// few queries the split tensor-core kernel stays ahead (decode, 64 or 256
// sequences, k = 512 or 2048: 21-32 us against 21-48 us).  The fused query
// prologue and output de-rotation exist only in the tensor-core kernel.
constexpr int64_t kTcMinRows = 257;
constexpr int kFewHeads = 16;
constexpr int64_t kManyQueries = 2048;
// CTAs of at most this many warps use 32-row tiles
constexpr int kSmallTileMaxWarps = 1;
bool attention_uses_tc(const AttnArgs& a) {
  const int32_t choice = attention_kernel_choice();
  if (choice == 2 || !tc_attention_supported(a)) return false;
  if (choice == 1) return true;
  if (a.qprologue || a.out_derotate) return true;
  const int64_t rows = (a.idx ? (int64_t)a.top_k : a.max_entries) + a.window;
  if (rows < kTcMinRows) return false;
  return !(a.H <= kFewHeads && a.T >= kManyQueries);
}

cudaError_t launch_attention(const Launch& L, const AttnArgs& a) {
  if (a.T == 0) return cudaSuccess;
  if (a.d == 512) {   // the pages' entry width (attention512.cu)
    L.begin(kKernelAttention);
    cudaError_t e = launch_attention512(L, a);
    if (e != cudaSuccess) return e;
    e = L.end(kKernelAttention);
    if (e != cudaSuccess || a.n_split == 1) return e;
    return launch_merge(L, a);
  }
  if (a.use_tc) {
    L.begin(kKernelAttention);
    AttnArgs b = a;
    if (take_attention_timeout_test()) {
      b.withhold_q = 1;
      b.wait_limit = 1ll << 21;
    }
    cudaError_t e = launch_attention_tc(L, b);
    if (e != cudaSuccess) return e;
    e = L.end(kKernelAttention);
    if (e != cudaSuccess || a.n_split == 1) return e;
    return launch_merge(L, a);
  }
  const int nw = a.H >= 64 ? 4 : (a.H + 15) / 16;
  const int hgroups = (a.H + nw * 16 - 1) / (nw * 16);
  const dim3 grid((unsigned)a.T, (unsigned)a.n_split, (unsigned)hgroups);
  const bool small = nw <= kSmallTileMaxWarps;
  L.begin(kKernelAttention);
  switch (nw) {
    case 1:
      if (small) attn_kernel<1, 32><<<grid, 32, 0, L.stream>>>(a);
      else attn_kernel<1, 64><<<grid, 32, 0, L.stream>>>(a);
      break;
    case 2:
      if (small) attn_kernel<2, 32><<<grid, 64, 0, L.stream>>>(a);
      else attn_kernel<2, 64><<<grid, 64, 0, L.stream>>>(a);
      break;
    case 3:
      if (small) attn_kernel<3, 32><<<grid, 96, 0, L.stream>>>(a);
      else attn_kernel<3, 64><<<grid, 96, 0, L.stream>>>(a);
      break;
    default:
      if (small) attn_kernel<4, 32><<<grid, 128, 0, L.stream>>>(a);
      else attn_kernel<4, 64><<<grid, 128, 0, L.stream>>>(a);
      break;
  }
  cudaError_t e = L.end(kKernelAttention);
  if (e != cudaSuccess || a.n_split == 1) return e;
  return launch_merge(L, a);
}

}  // namespace csa
