// 4-bit lightning indexer: quantization of indexer queries / keys to E2M1
// codes with one power-of-two scale byte per 32 elements, and indexer scoring
// straight from those codes.
//
// DeepSeek-V4 book, Ch.8 "A Cost Model for Long Context": "V4 compressed-entry
// payload" (the indexer key is cached in FP4, half a byte per scalar) and
// "Quantization scales and bounded tail buffers" (one 1-byte scale factor per
// 32 elements); Ch.6 "Top-k selection and asymptotic scaling" (the indexer
// scan runs in FP4).  The pages fix neither the element encoding nor the
// scale rule; the format here is the OCP Microscaling one:
//   * element: E2M1 (sign, 2 exponent bits with bias 1, 1 mantissa bit):
//     magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6;
//   * scale: byte b means 2^(b-127); for a block with largest magnitude amax,
//     b - 127 = floor(log2 amax) - 2, clamped to [-127, 127] (-127 for an
//     all-zero block);
//   * element code: x / 2^(b-127) rounded to the nearest magnitude, ties to
//     the even code, saturating at 6; the sign bit is x's sign bit;
//   * packing: byte i holds element 2i (low nibble) and 2i+1 (high nibble);
//     a vector of n elements is n/2 code bytes and n/32 scale bytes, the
//     scales in an array of their own with the same row order.
//
// Scoring uses the score definition of Ch.6 "The lightning indexer" on the
// dequantized values.  E2M1 magnitudes are exact fp16 numbers, so code bytes
// become fp16 pairs by sm_100a's e2m1x2 conversion; the tensor cores (mma.sync,
// fp16 inputs, fp32 accumulation) form the dot product of each 32-element
// scale block exactly (products are multiples of 1/4 below 36, sums below
// 1152), and the block results are scaled by 2^(b_q - 127) * 2^(b_k - 127)
// in fp32 before they are added.  The scorer is HBM-bound on the codes: 34
// bytes per 64-dim key instead of 128.  Keys leave as the same
// order-preserving 32-bit keys as the bf16 scorer (appended to the candidate
// lists), so the top-k selection is shared.
#include "kernels.h"
#include "lowprec.cuh"

namespace csa {

namespace {

// ---------------------------------------------------------------------------
// quantization: one thread per 32-element block
// ---------------------------------------------------------------------------
constexpr int kQuantThreads = 256;

using lowprec::quantize_block;

__global__ void __launch_bounds__(kQuantThreads) mxfp4_quantize_kernel(
    const __nv_bfloat16* __restrict__ x, int64_t n_blocks, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ scales) {
  const int64_t b = (int64_t)blockIdx.x * kQuantThreads + threadIdx.x;
  if (b >= n_blocks) return;
  uint32_t out[4];
  const uint32_t sb = quantize_block(x + b * 32, out);
  *reinterpret_cast<uint4*>(codes + b * 16) = make_uint4(out[0], out[1], out[2], out[3]);
  scales[b] = (uint8_t)sb;
}

// ---------------------------------------------------------------------------
// scoring
// ---------------------------------------------------------------------------
constexpr int kFp4Warps = 8;
constexpr int kFp4Threads = kFp4Warps * 32;
// 16-key groups per register batch (two batches in flight per warp): about
// 16 code bytes per lane per group at c_I = 64, fewer groups where the query
// fragments take more registers
constexpr int fp4_unroll(int ci, int nt) { return (ci == 64 ? 4 : 2) / (nt >= 4 ? 2 : 1); }

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                              uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Eight E2M1 codes (nibble j = element j) -> fp16 pairs (0,1), (2,3), (4,5),
// (6,7): every E2M1 value is an fp16 number, and sm_100a converts a byte of
// two codes (low nibble -> low half) in one instruction.
__device__ __forceinline__ uint4 e2m1x8_to_f16(uint32_t x) {
  uint4 r;
  asm("{\n"
      ".reg .b8 b0, b1, b2, b3;\n"
      "mov.b32 {b0, b1, b2, b3}, %4;\n"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n"
      "}\n"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "r"(x));
  return r;
}

// 2^(b - 127) for a scale byte b (b = 0: 2^-127, a subnormal)
__device__ __forceinline__ float e8m0_value(uint32_t b) {
  return b ? __uint_as_float(b << 23) : __uint_as_float(0x00400000u);
}

// Per-lane query data, identical in every warp: lane (g, q) holds, for each
// group of 8 heads nt and scale block v, the fp16 B fragments of head
// nt*8 + g over dims [32v + 8q, 32v + 8q + 8), the scale factors of heads
// nt*8 + 2q and nt*8 + 2q + 1 (the accumulator columns of the lane) and their
// weights.  Heads >= H_I are zero.
template <int CI, int NT>
struct Fp4Query {
  uint4 frag[NT][CI / 32][32];
  float2 fac[NT][CI / 32][32];
  float2 w[NT][32];
};

// Code words and scale bytes of kU 16-key groups: rows g (h = 0) and g + 8
// (h = 1) of each group, for lane (g, q).
template <int CI, int kU>
struct KeyBatch {
  uint32_t kw[kU][2][CI / 32];
  uint32_t ks[kU][2];
};

// base >= 0: contiguous cache whose rows base + [s_begin, s_end) were checked
// once for the whole chunk; else every row goes through cache_row.
template <int CI, int kU>
__device__ __forceinline__ void load_batch(KeyBatch<CI, kU>& kb, const IndexerArgs& a,
                                           const uint8_t* codes, int32_t seq, int64_t base,
                                           int64_t s0, int64_t s_end, int64_t t, int g, int q4) {
  constexpr int KB = CI / 32;
#pragma unroll
  for (int u = 0; u < kU; ++u) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t s = s0 + u * 16 + g + 8 * h;
      int64_t row = -1;
      if (s < s_end) row = base >= 0 ? base + s : cache_row(a.keys, seq, s, a.err, (int32_t)t);
      const uint32_t* rw =
          reinterpret_cast<const uint32_t*>(codes + (row >= 0 ? row : 0) * (CI / 2));
#pragma unroll
      for (int v = 0; v < KB; ++v) kb.kw[u][h][v] = row >= 0 ? __ldg(rw + 4 * v + q4) : 0u;
      if (CI == 64)
        kb.ks[u][h] =
            row >= 0 ? (uint32_t)__ldg(reinterpret_cast<const uint16_t*>(a.k_scales) + row) : 0u;
      else
        kb.ks[u][h] = row >= 0 ? __ldg(reinterpret_cast<const uint32_t*>(a.k_scales) + row) : 0u;
    }
  }
}

// The contraction dimension is permuted so that lane (g, q) of a key row
// needs only 32-bit word 4v + q of the row's codes for scale block v (dims
// [32v + 8q, 32v + 8q + 8)); the query fragments use the same permutation,
// which leaves every dot product unchanged, and every k-column of the two
// mma of block v falls inside block v.
template <int CI, int NT, int kU>
__device__ __forceinline__ void score_batch(const KeyBatch<CI, kU>& kb,
                                            const Fp4Query<CI, NT>& sq, const IndexerArgs& a,
                                            int64_t tl, uint32_t tau,
                                            CandidateBatch<kU>& pend, int64_t s0, int64_t s_end,
                                            int lane, int g, int q4) {
  bool pass[kU];
  uint32_t keys[kU], ents[kU];
  constexpr int KB = CI / 32;
#pragma unroll
  for (int u = 0; u < kU; ++u) {
    uint4 ka[2][KB];
    float fk[2][KB];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int v = 0; v < KB; ++v) {
        ka[h][v] = e2m1x8_to_f16(kb.kw[u][h][v]);
        fk[h][v] = e8m0_value((kb.ks[u][h] >> (8 * v)) & 0xffu);
      }
    float sg = 0.f, s8 = 0.f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float dg0 = 0.f, dg1 = 0.f, d80 = 0.f, d81 = 0.f;   // rows g / g+8, heads h0 / h0+1
#pragma unroll
      for (int v = 0; v < KB; ++v) {
        const uint4 bq = sq.frag[nt][v][lane];
        float d[4] = {0.f, 0.f, 0.f, 0.f};
        const uint32_t lo[4] = {ka[0][v].x, ka[1][v].x, ka[0][v].y, ka[1][v].y};
        mma_f16_16816(d, lo, bq.x, bq.y);
        const uint32_t hi[4] = {ka[0][v].z, ka[1][v].z, ka[0][v].w, ka[1][v].w};
        mma_f16_16816(d, hi, bq.z, bq.w);
        const float2 fq = sq.fac[nt][v][lane];
        dg0 += d[0] * fq.x * fk[0][v];
        dg1 += d[1] * fq.y * fk[0][v];
        d80 += d[2] * fq.x * fk[1][v];
        d81 += d[3] * fq.y * fk[1][v];
      }
      const float2 wv = sq.w[nt][lane];
      sg = fmaf(wv.x, fmaxf(dg0, 0.f), sg);
      sg = fmaf(wv.y, fmaxf(dg1, 0.f), sg);
      s8 = fmaf(wv.x, fmaxf(d80, 0.f), s8);
      s8 = fmaf(wv.y, fmaxf(d81, 0.f), s8);
    }
    sg += __shfl_xor_sync(0xffffffffu, sg, 1);
    s8 += __shfl_xor_sync(0xffffffffu, s8, 1);
    sg += __shfl_xor_sync(0xffffffffu, sg, 2);
    s8 += __shfl_xor_sync(0xffffffffu, s8, 2);
    const int64_t s = s0 + u * 16 + g + (q4 == 1 ? 8 : 0);
    const bool valid = q4 < 2 && s < s_end;
    keys[u] = score_key(q4 == 0 ? sg : s8);
    ents[u] = (uint32_t)s;
    pass[u] = valid && keys[u] >= tau;
  }
  CandidateBatch<kU> cur;
  cur.issue(a, tl, pass, keys, ents);
  pend.flush(a);
  pend = cur;
}

// One CTA scores a chunk of one query's keys.  The prologue quantizes the
// query's bf16 heads (the same block quantizer as csa_quantize_mxfp4) and
// lays out its fragments; each warp then walks batches of kU 16-key groups,
// loading the next batch's code words into the other register set before it
// scores the current one.
template <int CI, int NT>
__global__ void __launch_bounds__(kFp4Threads, (CI == 64 && NT == 1) ? 3 : 1)
indexer_score_fp4_kernel(IndexerArgs a, int64_t chunk) {
  constexpr int KB = CI / 32;                  // scale blocks per vector
  constexpr int kU = fp4_unroll(CI, NT);       // 16-key groups per batch
  __shared__ Fp4Query<CI, NT> sq;
  __shared__ uint32_t qwords[NT * 8][CI / 8];  // the query's codes, head-major
  __shared__ uint32_t qscale[NT * 8][KB];
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
  for (int i = threadIdx.x; i < a.H_I * KB; i += kFp4Threads) {
    const int h = i / KB, v = i - h * KB;
    uint32_t w4[4];
    qscale[h][v] = quantize_block(a.q_idx + (t * a.H_I + h) * CI + 32 * v, w4);
#pragma unroll
    for (int j = 0; j < 4; ++j) qwords[h][4 * v + j] = w4[j];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < NT * KB * 32; i += kFp4Threads) {
    const int L = i & 31, v = (i >> 5) % KB, nt = (i >> 5) / KB;
    const int hg = nt * 8 + (L >> 2), h0 = nt * 8 + 2 * (L & 3);
    sq.frag[nt][v][L] = e2m1x8_to_f16(hg < a.H_I ? qwords[hg][4 * v + (L & 3)] : 0u);
    const float f0 = h0 < a.H_I ? e8m0_value(qscale[h0][v]) : 0.f;
    const float f1 = h0 + 1 < a.H_I ? e8m0_value(qscale[h0 + 1][v]) : 0.f;
    sq.fac[nt][v][L] = make_float2(f0, f1);
    if (v == 0)
      sq.w[nt][L] = make_float2(h0 < a.H_I ? __ldg(a.w + t * a.H_I + h0) : 0.f,
                                h0 + 1 < a.H_I ? __ldg(a.w + t * a.H_I + h0 + 1) : 0.f);
  }
  __syncthreads();

  const uint8_t* codes = reinterpret_cast<const uint8_t*>(a.keys.data);
  const uint32_t tau = __ldg(a.tau + tl);
  CandidateBatch<kU> pend;   // the previous batch's candidates
  const int64_t stride = (int64_t)kFp4Warps * 16 * kU;
  // a contiguous cache whose chunk lies inside the buffer skips the per-row
  // checks (the same conditions cache_row tests, once for the whole chunk)
  int64_t base = -1;
  if (a.keys.page_table == nullptr) {
    const int64_t b = (int64_t)seq * a.keys.seq_stride;
    if (b >= 0 && (a.keys.seq_stride == 0 || s_end <= a.keys.seq_stride) && b + s_end <= a.keys.n_rows)
      base = b;
  }
  KeyBatch<CI, kU> b0, b1;
  int64_t s0 = s_begin + (int64_t)warp * 16 * kU;
  if (s0 < s_end) load_batch(b0, a, codes, seq, base, s0, s_end, t, g, q4);
  while (s0 < s_end) {
    int64_t s1 = s0 + stride;
    if (s1 < s_end) load_batch(b1, a, codes, seq, base, s1, s_end, t, g, q4);
    score_batch<CI, NT>(b0, sq, a, tl, tau, pend, s0, s_end, lane, g, q4);
    if (s1 >= s_end) break;
    s0 = s1 + stride;
    if (s0 < s_end) load_batch(b0, a, codes, seq, base, s0, s_end, t, g, q4);
    score_batch<CI, NT>(b1, sq, a, tl, tau, pend, s1, s_end, lane, g, q4);
  }
  pend.flush(a);
}

template <int CI, int NT>
void launch_score_fp4(const Launch& L, const IndexerArgs& a, int64_t t_count) {
  constexpr int kU = fp4_unroll(CI, NT);
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, indexer_score_fp4_kernel<CI, NT>,
                                                kFp4Threads, 0);
  if (per_sm < 1) per_sm = 1;
  // chunks per query so that the grid fills whole resident waves
  const int64_t wave = (int64_t)sms * per_sm;
  int64_t per_q = wave / t_count;
  if (per_q < 1) per_q = 1;
  const int64_t min_chunk = 16 * kFp4Warps * kU;   // one pass of the warps
  int64_t chunk = (a.max_entries + per_q - 1) / per_q;
  chunk = (chunk + min_chunk - 1) / min_chunk * min_chunk;
  if (chunk < min_chunk) chunk = min_chunk;
  per_q = (a.max_entries + chunk - 1) / chunk;
  const dim3 grid((unsigned)t_count, (unsigned)per_q);
  prefer_max_shared(indexer_score_fp4_kernel<CI, NT>);
  indexer_score_fp4_kernel<CI, NT><<<grid, kFp4Threads, 0, L.stream>>>(a, chunk);
}

}  // namespace

cudaError_t launch_mxfp4_quantize(const Launch& L, const __nv_bfloat16* x, int64_t n_blocks,
                                  uint8_t* codes, uint8_t* scales) {
  if (n_blocks == 0) return cudaSuccess;
  L.begin(kKernelQuantize);
  const unsigned blocks = (unsigned)((n_blocks + kQuantThreads - 1) / kQuantThreads);
  mxfp4_quantize_kernel<<<blocks, kQuantThreads, 0, L.stream>>>(x, n_blocks, codes, scales);
  return L.end(kKernelQuantize);
}

cudaError_t launch_indexer_scores_fp4(const Launch& L, const IndexerArgs& a, int64_t t_count) {
  if (t_count == 0 || a.max_entries == 0) return cudaSuccess;
  const int nt = (a.H_I + 7) / 8;
  const int ntb = nt <= 1 ? 1 : nt <= 2 ? 2 : nt <= 4 ? 4 : 8;
  L.begin(kKernelIndexerScore);
#define CSA_FP4_CASE(CI_, NT_) \
  if (a.c_I == CI_ && ntb == NT_) launch_score_fp4<CI_, NT_>(L, a, t_count);
  CSA_FP4_CASE(64, 1)
  CSA_FP4_CASE(64, 2)
  CSA_FP4_CASE(64, 4)
  CSA_FP4_CASE(64, 8)
  CSA_FP4_CASE(128, 1)
  CSA_FP4_CASE(128, 2)
  CSA_FP4_CASE(128, 4)
  CSA_FP4_CASE(128, 8)
#undef CSA_FP4_CASE
  return L.end(kKernelIndexerScore);
}

}  // namespace csa
