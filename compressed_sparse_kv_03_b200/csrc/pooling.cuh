// Coordinate-wise softmax pooling of m source rows, shared by the bulk
// compressor and the decode-time cache append so that both produce the same
// bits for the same block.
//
// DeepSeek-V4 book, Ch.5 "Coordinate-wise softmax pooling": per coordinate r
// a softmax over the pooled tokens' logits weights their content.  One thread
// owns 8 consecutive coordinates (one 16-byte vector per source row); the
// softmax runs online in fp32 (log2 domain) over chunks of 4 rows, the 8
// loads of a chunk issued before any arithmetic.
#pragma once

#include "kernels.h"

namespace csa {
namespace pooling {

constexpr int kChunk = 4;

struct Acc8 {
  float mx[8], sum[8], acc[8];
};

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  float2 a = unpack_bf16(v.x), b = unpack_bf16(v.y), c = unpack_bf16(v.z), d = unpack_bf16(v.w);
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y; f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}

// Pool rows row0 .. row0+m-1 of (C, Z) into the running accumulator; the bias
// row for source j is bias[(j - row0) * dim].  kStream: read-only streaming
// loads (rows not written by the running kernel); else plain coherent loads,
// for rows the calling thread has just written (C and Z are deliberately not
// __restrict__, which would let the compiler turn those loads into
// non-coherent read-only ones).
template <bool kStream>
__device__ __forceinline__ void pool_rows(Acc8& A, const __nv_bfloat16* C, const __nv_bfloat16* Z,
                                          const float* __restrict__ bias, int64_t row0, int m,
                                          int dim, int c0) {
  for (int j0 = 0; j0 < m; j0 += kChunk) {
    uint4 cv[kChunk], zv[kChunk];
#pragma unroll
    for (int r = 0; r < kChunk; ++r) {
      if (j0 + r < m) {
        const int64_t off = (row0 + j0 + r) * (int64_t)dim + c0;
        if (kStream) {
          cv[r] = ld_stream_16(C + off);
          zv[r] = ld_stream_16(Z + off);
        } else {
          cv[r] = *reinterpret_cast<const uint4*>(C + off);
          zv[r] = *reinterpret_cast<const uint4*>(Z + off);
        }
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

__device__ __forceinline__ void init(Acc8& A) {
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    A.mx[e] = -INFINITY;
    A.sum[e] = 0.f;
    A.acc[e] = 0.f;
  }
}

__device__ __forceinline__ uint4 finish(const Acc8& A) {
  uint4 o;
  o.x = pack_bf16(A.acc[0] / A.sum[0], A.acc[1] / A.sum[1]);
  o.y = pack_bf16(A.acc[2] / A.sum[2], A.acc[3] / A.sum[3]);
  o.z = pack_bf16(A.acc[4] / A.sum[4], A.acc[5] / A.sum[5]);
  o.w = pack_bf16(A.acc[6] / A.sum[6], A.acc[7] / A.sum[7]);
  return o;
}

}  // namespace pooling
}  // namespace csa
