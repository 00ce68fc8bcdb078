// Attention prologue / epilogue: RMSNorm and partial RoPE, or the output
// de-rotation.
//
// DeepSeek-V4 book, Ch.2 "Normalization and rotary position embeddings" and
// Ch.7 "Query and KV RMSNorm", "Partial RoPE and output de-rotation": every
// query head and every shared KV vector is RMS-normalised (times a learned
// gain) before the dot products; the last 64 coordinates are rotated by the
// block-diagonal R_t of their position; the attention output's rotary
// coordinates get R_{-t} of the query position.  Pairs (2j, 2j+1) of the
// rotary slice turn by t * base^(-2j / rope_dims).
//
// HBM-bound elementwise pass: 16 threads per 128-dim vector (one 16-byte
// vector each), the sum of squares reduced over the 16 lanes; a thread walks
// 8 heads of one position, so their rotation is computed once; rotation angles
// are formed and reduced modulo 2 pi in double precision from frequencies the
// host computes (positions reach 2^20 and more, beyond what an fp32 angle
// resolves), then sin / cos in fp32.
#include <cmath>

#include "kernels.h"

namespace csa {

namespace {

constexpr int kThreads = 256;

constexpr int kHeadsPerThread = 8;   // heads of one position sharing the rotation

__global__ void __launch_bounds__(kThreads) norm_rope_kernel(NormRopeArgs a) {
  const int lanes = a.dim >> 3;                      // threads per vector (power of two)
  const int hgroups = (a.H + kHeadsPerThread - 1) / kHeadsPerThread;
  const int64_t gid = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  const int64_t grp = gid / lanes;                   // (t, head group)
  const int sub = (int)(gid - grp * lanes);
  const bool live = grp < a.T * hgroups;
  const int64_t t = live ? grp / hgroups : 0;
  const int h0 = live ? (int)(grp - t * hgroups) * kHeadsPerThread : 0;
  const int c0 = sub * 8;
  const int r0 = a.dim - a.rope_dims;
  const bool rot = live && a.rope_dims > 0 && c0 >= r0;
  // this thread's four pair rotations, shared by its heads
  float cs[4] = {1.f, 1.f, 1.f, 1.f}, sn[4] = {0.f, 0.f, 0.f, 0.f};
  if (rot) {
    const int64_t p = (a.pos ? __ldg(a.pos + t) : t) * a.pos_mul;
    const double two_pi = 6.283185307179586476925, inv_two_pi = 0.159154943091895335769;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = ((c0 - r0) >> 1) + e;
      double ang = (double)p * a.theta[j];
      ang -= two_pi * floor(ang * inv_two_pi);   // into [0, 2 pi)
      if (a.inverse) ang = -ang;
      sincosf((float)ang, &sn[e], &cs[e]);
    }
  }
  float g[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) g[e] = 1.f;
  if (a.gain != nullptr && a.eps >= 0.f) {
    const float4 g0 = __ldg(reinterpret_cast<const float4*>(a.gain + c0));
    const float4 g1 = __ldg(reinterpret_cast<const float4*>(a.gain + c0 + 4));
    g[0] = g0.x; g[1] = g0.y; g[2] = g0.z; g[3] = g0.w; g[4] = g1.x; g[5] = g1.y; g[6] = g1.z; g[7] = g1.w;
  }
#pragma unroll 4
  for (int hh = 0; hh < kHeadsPerThread; ++hh) {
    const int h = h0 + hh;
    const bool on = live && h < a.H;                  // uniform over the vector's lanes
    const int64_t vec = t * a.H + h;
    float x[8];
    if (on) {
      const uint4 v = *reinterpret_cast<const uint4*>(a.x + vec * a.dim + c0);
      const float2 p0 = unpack_bf16(v.x), p1 = unpack_bf16(v.y), p2 = unpack_bf16(v.z), p3 = unpack_bf16(v.w);
      x[0] = p0.x; x[1] = p0.y; x[2] = p1.x; x[3] = p1.y; x[4] = p2.x; x[5] = p2.y; x[6] = p3.x; x[7] = p3.y;
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = 0.f;
    }
    if (a.eps >= 0.f) {
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) ss = fmaf(x[e], x[e], ss);
      for (int o = lanes >> 1; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float r = rsqrtf(ss / (float)a.dim + a.eps);
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] *= r * g[e];
    }
    if (rot) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float u = x[2 * e], w = x[2 * e + 1];
        x[2 * e] = u * cs[e] - w * sn[e];
        x[2 * e + 1] = u * sn[e] + w * cs[e];
      }
    }
    if (on) {
      uint4 o;
      o.x = pack_bf16(x[0], x[1]);
      o.y = pack_bf16(x[2], x[3]);
      o.z = pack_bf16(x[4], x[5]);
      o.w = pack_bf16(x[6], x[7]);
      *reinterpret_cast<uint4*>(a.out + vec * a.dim + c0) = o;
    }
  }
}

}  // namespace

cudaError_t launch_norm_rope(const Launch& L, const NormRopeArgs& args) {
  const int64_t threads = args.T * ((args.H + kHeadsPerThread - 1) / kHeadsPerThread) * (args.dim >> 3);
  if (threads == 0) return cudaSuccess;
  NormRopeArgs a = args;
  for (int j = 0; j < a.rope_dims / 2; ++j)
    a.theta[j] = std::pow((double)a.rope_base, -2.0 * j / (double)a.rope_dims);
  L.begin(kKernelCompress);
  norm_rope_kernel<<<(unsigned)((threads + kThreads - 1) / kThreads), kThreads, 0, L.stream>>>(a);
  return L.end(kKernelCompress);
}

}  // namespace csa
