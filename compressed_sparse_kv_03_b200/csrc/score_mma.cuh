// Tensor-core (mma.sync) scoring of 16-key groups against a query's indexer
// heads: the scorer of indexer.cu and the fused selection's sample pass use
// the same fragments and the same arithmetic.
//
// Keys sit on the MMA M dimension (16 rows), heads on N (8 per tile), the key
// dim is K.  The contraction dimension is permuted so that every lane reads
// whole 16-byte vectors of a key row: lane (g, q) holds dims
// [32v + 8q, 32v + 8q + 8) of rows g and g+8; the query fragments are loaded
// with the same permutation, which leaves every dot product unchanged.
#pragma once

#include "kernels.h"

namespace csa {

// Query fragments of lane (g, q) for NT tiles of 8 heads, and the lane's two
// head weights per tile (heads >= H_I are zero).
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

}  // namespace csa
