// Step 4 at head dim 512: shared-KV softmax attention over gathered rows for
// the pages' entry width (DeepSeek-V4 book, Ch.6 "Shared key-value MQA",
// Ch.7 "The 128-token uncompressed sliding window", "Dense attention over
// heavily compressed history"; Ch.5 "Decode-time cache state" for c = 512).
//
// The same virtual row list, split-KV slices and online softmax as the d = 128
// mma.sync kernel (attention.cu), laid out for 512-dim rows.  A CTA takes one
// query, one slice and 32 heads: two groups of 16 heads, four warps each,
// sharing every tile of rows.  Warp w of a group owns dims [128 w, 128 w +
// 128): it contracts its quarter of Q K^T for the tile (mma.sync m16n8k16,
// bf16 in, fp32 accumulate), the group's four partial score tiles are summed
// through shared memory in a fixed order (all four warps then hold the same
// scores and run the same online softmax), and it accumulates O for its own
// dims.  Rows arrive 32 at a time by cp.async into a double-buffered,
// XOR-swizzled tile (2 x 32 KB); the query's heads sit in shared memory
// (32 KB) and are read as MMA fragments per step, so that a thread stays
// within 128 registers and two CTAs share an SM.
#include "kernels.h"

namespace csa {

namespace {

constexpr int kD5 = 512;         // head dim
constexpr int kBN5 = 32;         // rows per tile
static_assert(kBN5 == 32, "one 32-bit validity word per stage; fragments of kBN5 / 8 n-tiles");
constexpr int kQ5 = 4;           // warps per head group; warp w owns dims [kDW5 w, kDW5 (w + 1))
constexpr int kG5 = 2;           // head groups of 16 per CTA
constexpr int kW5 = kQ5 * kG5;   // warps
constexpr int kDW5 = kD5 / kQ5;  // 128
constexpr int kHeads5 = 16 * kG5;   // heads per CTA
constexpr int kSw5 = kBN5 / 2;   // floats per lane in the score exchange (kBN5 / 8 fragments of 4)
constexpr size_t kQOff5 = 2 * kBN5 * kD5 * sizeof(__nv_bfloat16);
constexpr size_t kSOff5 = kQOff5 + kHeads5 * kD5 * sizeof(__nv_bfloat16);
constexpr size_t kSmem5 = kSOff5 + kW5 * 32 * kSw5 * sizeof(float);   // 112 KB: two CTAs per SM

__global__ void __launch_bounds__(kW5 * 32, 2) attn512_kernel(AttnArgs a) {
  constexpr int NTH = kW5 * 32;
  extern __shared__ __align__(128) uint8_t smem5[];
  __nv_bfloat16* const sKV = reinterpret_cast<__nv_bfloat16*>(smem5);                   // 2 x kBN5 x kD5
  __nv_bfloat16* const sQ = reinterpret_cast<__nv_bfloat16*>(smem5 + kQOff5);          // kHeads5 x kD5
  float* const sS = reinterpret_cast<float*>(smem5 + kSOff5);
  __shared__ const __nv_bfloat16* sRow[2][kBN5];
  __shared__ uint32_t sMask[2][kBN5 / 32];   // row validity bits of each stage

  const int64_t i = blockIdx.x;
  const int split = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, q4 = lane & 3;
  const int hgrp = warp / kQ5, dq = warp % kQ5;
  const int head0 = blockIdx.z * kHeads5 + 16 * hgrp;
  const int dw0 = dq * kDW5;
  const bool reporter = split == 0 && tid == 0 && blockIdx.z == 0;

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
      if (reporter) report(a.err, kErrEligible, (int32_t)i, n_sel);
      n_sel = a.max_entries;
    }
  }
  int64_t n_win, win_first = 0;
  if (a.win_len) {
    n_win = __ldg(a.win_len + i);
    if (n_win < 0 || n_win > a.window) {
      if (reporter) report(a.err, kErrWindow, (int32_t)i, n_win);
      n_win = n_win < 0 ? 0 : a.window;
    }
  } else {
    win_first = attn_raw_window(a, i, pos, n_win, reporter);
  }
  const int64_t total = n_sel + n_win;
  const int64_t v0 = (int64_t)split * a.split_len;
  const int64_t v1 = total < v0 + a.split_len ? total : v0 + a.split_len;
  const int ntiles = v1 > v0 ? (int)((v1 - v0 + kBN5 - 1) / kBN5) : 0;

  auto fill_rows = [&](int st, int tt) {
    for (int r0 = warp * 32; r0 < kBN5; r0 += NTH) {
      const int r = r0 + lane;
      const int64_t v = v0 + (int64_t)tt * kBN5 + r;
      const __nv_bfloat16* p = nullptr;
      if (v < v1) {
        if (v < n_sel) {
          const int64_t e = a.idx ? (int64_t)__ldg(a.idx + i * a.top_k + v) : v;
          const int64_t rr = cache_row(a.kv, seq, e, a.err, (int32_t)i);
          if (rr >= 0) p = a.kv.data + rr * kD5;
        } else {
          const int64_t w = v - n_sel;
          p = a.win_len ? a.win + (i * a.window + w) * kD5 : a.win + (win_first + w) * kD5;
        }
      }
      sRow[st][r] = p;
      const uint32_t bits = __ballot_sync(0xffffffffu, p != nullptr);
      if (lane == 0) sMask[st][r0 >> 5] = bits;
    }
  };
  // row r's 16-byte chunk ch at r * kD5 + 8 (ch ^ (r mod 8)) elements
  auto issue_tile = [&](int st) {
    const uint32_t base = smem_u32(sKV + st * kBN5 * kD5);
    for (int c = tid; c < kBN5 * (kD5 / 8); c += NTH) {
      const int r = c / (kD5 / 8), ch = c % (kD5 / 8);
      const __nv_bfloat16* src = sRow[st][r];
      const uint32_t off = (uint32_t)(r * kD5 + ((ch ^ (r & 7)) << 3));
      cp_async_16(base + off * 2u, src ? src + ch * 8 : a.q, src != nullptr);
    }
  };

  // ---- the CTA's 32 heads of the query in shared memory: head h's 16-byte
  // chunk ch at h * kD5 + 8 (ch ^ (h mod 8)) elements (zeros past H) ----
  for (int c = tid; c < kHeads5 * (kD5 / 8); c += NTH) {
    const int hh = c / (kD5 / 8), ch = c % (kD5 / 8);
    const int h = blockIdx.z * kHeads5 + hh;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (h < a.H) v = *reinterpret_cast<const uint4*>(a.q + (i * a.H + h) * kD5 + ch * 8);
    *reinterpret_cast<uint4*>(sQ + hh * kD5 + ((ch ^ (hh & 7)) << 3)) = v;
  }
  const float scale = a.sm_scale * kLog2e;

  float acc[kDW5 / 8][4];
#pragma unroll
  for (int n = 0; n < kDW5 / 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
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

    const uint32_t sbase = smem_u32(sKV + st * kBN5 * kD5);
    // this warp's quarter of S = Q K^T (16 heads x 64 rows)
    float s[kBN5 / 8][4];
#pragma unroll
    for (int j = 0; j < kBN5 / 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
    const uint32_t qbase = smem_u32(sQ);
#pragma unroll
    for (int kk = 0; kk < kDW5 / 16; ++kk) {
      uint32_t qa[4];   // heads 16 hgrp + (0..15) x dims dw0 + 16 kk + (0..15)
      {
        const int hr = 16 * hgrp + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int ch = dw0 / 8 + 2 * kk + (lane >> 4);
        ldmatrix_x4(qa, qbase + (uint32_t)(hr * kD5 + ((ch ^ (hr & 7)) << 3)) * 2u);
      }
#pragma unroll
      for (int jp = 0; jp < kBN5 / 16; ++jp) {
        const int mi = lane >> 3, rr = lane & 7;
        const int row = 16 * jp + 8 * (mi >> 1) + rr;
        const int ch = dw0 / 8 + 2 * kk + (mi & 1);
        uint32_t r[4];
        ldmatrix_x4(r, sbase + (uint32_t)(row * kD5 + ((ch ^ (row & 7)) << 3)) * 2u);
        mma_bf16_16816(s[2 * jp], qa, r[0], r[1]);
        mma_bf16_16816(s[2 * jp + 1], qa, r[2], r[3]);
      }
    }
    // the four quarters meet in shared memory (the same fragment layout in
    // every warp); every warp sums them in the same order, so all four hold
    // the same scores bit for bit
    {
      // lane l's four float4 slots in the order j ^ ((l >> 1) & 3): the eight
      // lanes of a 16-byte access phase then meet eight different banks
      const int xs = (lane >> 1) & 3;
      float* const mine = sS + (warp * 32 + lane) * kSw5;
#pragma unroll
      for (int j = 0; j < kBN5 / 8; ++j)
        *reinterpret_cast<float4*>(mine + 4 * (j ^ xs)) = make_float4(s[j][0], s[j][1], s[j][2], s[j][3]);
      __syncthreads();
#pragma unroll
      for (int j = 0; j < kBN5 / 8; ++j) {
        float4 t = *reinterpret_cast<const float4*>(sS + ((hgrp * kQ5 + 0) * 32 + lane) * kSw5 + 4 * (j ^ xs));
#pragma unroll
        for (int w2 = 1; w2 < kQ5; ++w2) {
          const float4 u = *reinterpret_cast<const float4*>(sS + ((hgrp * kQ5 + w2) * 32 + lane) * kSw5 + 4 * (j ^ xs));
          t.x += u.x;
          t.y += u.y;
          t.z += u.z;
          t.w += u.w;
        }
        s[j][0] = t.x;
        s[j][1] = t.y;
        s[j][2] = t.z;
        s[j][3] = t.w;
      }
    }
    // online softmax (log2 domain); rows g (lo) and g + 8 (hi) are heads
    const uint32_t vmask = sMask[st][0];
    float mx_lo = -INFINITY, mx_hi = -INFINITY;
#pragma unroll
    for (int j = 0; j < kBN5 / 8; ++j) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const bool ok = (vmask >> (8 * j + 2 * q4 + c)) & 1u;
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
    for (int n = 0; n < kDW5 / 8; ++n) {
      acc[n][0] *= al_lo;
      acc[n][1] *= al_lo;
      acc[n][2] *= al_hi;
      acc[n][3] *= al_hi;
    }
    uint32_t pa[kBN5 / 16][4];
#pragma unroll
    for (int j = 0; j < kBN5 / 8; ++j) {
      const float p0 = exp2f(s[j][0] - ref_lo), p1 = exp2f(s[j][1] - ref_lo);
      const float p2 = exp2f(s[j][2] - ref_hi), p3 = exp2f(s[j][3] - ref_hi);
      l_lo += p0 + p1;
      l_hi += p2 + p3;
      pa[j >> 1][(j & 1) * 2 + 0] = pack_bf16(p0, p1);
      pa[j >> 1][(j & 1) * 2 + 1] = pack_bf16(p2, p3);
    }
    // O[:, this warp's dims] += P V
#pragma unroll
    for (int kk2 = 0; kk2 < kBN5 / 16; ++kk2) {
#pragma unroll
      for (int np = 0; np < kDW5 / 16; ++np) {
        const int mi = lane >> 3, rr = lane & 7;
        const int row = 16 * kk2 + 8 * (mi & 1) + rr;
        const int ch = dw0 / 8 + 2 * np + (mi >> 1);
        uint32_t r[4];
        ldmatrix_x4_trans(r, sbase + (uint32_t)(row * kD5 + ((ch ^ (row & 7)) << 3)) * 2u);
        mma_bf16_16816(acc[2 * np], pa[kk2], r[0], r[1]);
        mma_bf16_16816(acc[2 * np + 1], pa[kk2], r[2], r[3]);
      }
    }
    __syncthreads();   // stage st, sRow[st] and the score slots are reused
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
    for (int n = 0; n < kDW5 / 8; ++n) {
      const int c = dw0 + 8 * n + 2 * q4;
      if (h_lo < a.H)
        *reinterpret_cast<uint32_t*>(a.out + (i * a.H + h_lo) * kD5 + c) =
            pack_bf16(acc[n][0] * inv_lo, acc[n][1] * inv_lo);
      if (h_hi < a.H)
        *reinterpret_cast<uint32_t*>(a.out + (i * a.H + h_hi) * kD5 + c) =
            pack_bf16(acc[n][2] * inv_hi, acc[n][3] * inv_hi);
    }
    if (a.lse && q4 == 0 && dq == 0) {
      if (h_lo < a.H) a.lse[i * a.H + h_lo] = den_lo > 0.f ? (mm_lo + log2f(den_lo)) / kLog2e : -INFINITY;
      if (h_hi < a.H) a.lse[i * a.H + h_hi] = den_hi > 0.f ? (mm_hi + log2f(den_hi)) / kLog2e : -INFINITY;
    }
  } else {
    const int64_t pbase = (i * a.n_split + split) * a.H;
#pragma unroll
    for (int n = 0; n < kDW5 / 8; ++n) {
      const int c = dw0 + 8 * n + 2 * q4;
      if (h_lo < a.H)
        *reinterpret_cast<float2*>(a.part_acc + (pbase + h_lo) * kD5 + c) = make_float2(acc[n][0], acc[n][1]);
      if (h_hi < a.H)
        *reinterpret_cast<float2*>(a.part_acc + (pbase + h_hi) * kD5 + c) = make_float2(acc[n][2], acc[n][3]);
    }
    if (q4 == 0 && dq == 0) {
      if (h_lo < a.H) *reinterpret_cast<float2*>(a.part_ml + (pbase + h_lo) * 2) = make_float2(m_lo, l_lo);
      if (h_hi < a.H) *reinterpret_cast<float2*>(a.part_ml + (pbase + h_hi) * 2) = make_float2(m_hi, l_hi);
    }
  }
}

}  // namespace

cudaError_t launch_attention512(const Launch& L, const AttnArgs& a) {
  if (a.T == 0) return cudaSuccess;
  const dim3 grid((unsigned)a.T, (unsigned)a.n_split, (unsigned)((a.H + kHeads5 - 1) / kHeads5));
  cudaFuncSetAttribute(attn512_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem5);
  prefer_max_shared(attn512_kernel);
  attn512_kernel<<<grid, kW5 * 32, kSmem5, L.stream>>>(a);
  return cudaGetLastError();
}

}  // namespace csa
