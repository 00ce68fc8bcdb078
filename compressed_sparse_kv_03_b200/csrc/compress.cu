// Step 1: block compression by coordinate-wise softmax pooling.
//
// DeepSeek-V4 book, Ch.5 "How CSA Compresses Memory" ("Coordinate-wise softmax
// pooling": per coordinate r a softmax over the pooled source tokens, used to
// weight their content) and Ch.7 "HCA's 128:1 non-overlapping compressor".
//
// HBM-bound streaming reduction.  One thread owns one compressed entry and 8
// consecutive coordinates (one 16-byte vector of C and of Z per source row),
// so a warp reads whole 256-byte row segments: every load is a full, aligned
// 16-byte vector and each byte of C and Z is read exactly once.  The softmax
// runs online in fp32 (log2 domain) over chunks of 4 source rows: the 8 loads
// of a chunk are issued before any arithmetic, the running max is raised once
// per chunk, so there is about one exp2 per element.
#include "kernels.h"

namespace csa {

namespace {

constexpr int kChunk = 4;
constexpr int kThreads = 256;

struct Acc8 {
  float mx[8], sum[8], acc[8];
};

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  float2 a = unpack_bf16(v.x), b = unpack_bf16(v.y), c = unpack_bf16(v.z), d = unpack_bf16(v.w);
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y; f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}

// Pool rows row0 .. row0+m-1 of (C, Z) into the running accumulator; the bias
// row for source j is bias[(j - row0) * dim].
__device__ __forceinline__ void pool_rows(Acc8& A, const __nv_bfloat16* __restrict__ C,
                                          const __nv_bfloat16* __restrict__ Z,
                                          const float* __restrict__ bias, int64_t row0, int m,
                                          int dim, int c0) {
  for (int j0 = 0; j0 < m; j0 += kChunk) {
    uint4 cv[kChunk], zv[kChunk];
#pragma unroll
    for (int r = 0; r < kChunk; ++r) {
      if (j0 + r < m) {
        const int64_t off = (row0 + j0 + r) * (int64_t)dim + c0;
        cv[r] = ld_stream_16(C + off);
        zv[r] = ld_stream_16(Z + off);
      }
    }
    float u[kChunk][8], c[kChunk][8];
#pragma unroll
    for (int r = 0; r < kChunk; ++r) {
      if (j0 + r < m) {
        unpack8(cv[r], c[r]);
        unpack8(zv[r], u[r]);
        if (bias != nullptr) {
          const float4* bp = reinterpret_cast<const float4*>(bias + (int64_t)(j0 + r) * dim + c0);
          float4 b0 = __ldg(bp), b1 = __ldg(bp + 1);
          u[r][0] += b0.x; u[r][1] += b0.y; u[r][2] += b0.z; u[r][3] += b0.w;
          u[r][4] += b1.x; u[r][5] += b1.y; u[r][6] += b1.z; u[r][7] += b1.w;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) u[r][e] *= kLog2e;
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float cm = A.mx[e];
#pragma unroll
      for (int r = 0; r < kChunk; ++r)
        if (j0 + r < m) cm = fmaxf(cm, u[r][e]);
      // cm is finite: every pooled logit is finite
      const float scale = exp2f(A.mx[e] - cm);   // 0 when A.mx is -inf
      float s = A.sum[e] * scale, a = A.acc[e] * scale;
#pragma unroll
      for (int r = 0; r < kChunk; ++r) {
        if (j0 + r < m) {
          const float p = exp2f(u[r][e] - cm);
          s += p;
          a = fmaf(p, c[r][e], a);
        }
      }
      A.mx[e] = cm;
      A.sum[e] = s;
      A.acc[e] = a;
    }
  }
}

__global__ void __launch_bounds__(kThreads) compress_kernel(
    const __nv_bfloat16* __restrict__ Ca, const __nv_bfloat16* __restrict__ Za,
    const __nv_bfloat16* __restrict__ Cb, const __nv_bfloat16* __restrict__ Zb,
    const float* __restrict__ bias, int64_t S, int dim, int m, int overlap,
    __nv_bfloat16* __restrict__ out) {
  const int vecs = dim >> 3;
  const int64_t tid = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (tid >= S * vecs) return;
  const int64_t i = tid / vecs;
  const int c0 = (int)(tid - i * vecs) * 8;

  Acc8 A;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    A.mx[e] = -INFINITY;
    A.sum[e] = 0.f;
    A.acc[e] = 0.f;
  }
  // a branch: block i with (C_a, Z_a + bias[0])
  pool_rows(A, Ca, Za, bias, (int64_t)m * i, m, dim, c0);
  // b branch: block i-1 with (C_b, Z_b + bias[1]); block 0 has none
  if (overlap && i > 0)
    pool_rows(A, Cb, Zb, bias ? bias + (int64_t)m * dim : nullptr, (int64_t)m * (i - 1), m, dim,
              c0);

  uint4 o;
  o.x = pack_bf16(A.acc[0] / A.sum[0], A.acc[1] / A.sum[1]);
  o.y = pack_bf16(A.acc[2] / A.sum[2], A.acc[3] / A.sum[3]);
  o.z = pack_bf16(A.acc[4] / A.sum[4], A.acc[5] / A.sum[5]);
  o.w = pack_bf16(A.acc[6] / A.sum[6], A.acc[7] / A.sum[7]);
  *reinterpret_cast<uint4*>(out + i * dim + c0) = o;
}

}  // namespace

cudaError_t launch_compress(const Launch& L, const __nv_bfloat16* Ca, const __nv_bfloat16* Za,
                            const __nv_bfloat16* Cb, const __nv_bfloat16* Zb, const float* bias,
                            int64_t n_tokens, int dim, int m, int overlap, __nv_bfloat16* out) {
  const int64_t S = n_tokens / m;
  if (S == 0) return cudaSuccess;
  const int64_t threads = S * (dim / 8);
  const unsigned blocks = (unsigned)((threads + kThreads - 1) / kThreads);
  L.begin(kKernelCompress);
  compress_kernel<<<blocks, kThreads, 0, L.stream>>>(Ca, Za, Cb ? Cb : Ca, Zb ? Zb : Za, bias, S,
                                                     dim, m, overlap, out);
  return L.end(kKernelCompress);
}

}  // namespace csa
