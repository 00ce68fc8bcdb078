// Mixed-precision storage of compressed entries: the content coordinates as
// E4M3 codes with one power-of-two scale byte per 32, the trailing rotary
// coordinates kept in bf16.
//
// DeepSeek-V4 book, Ch.8 "A Cost Model for Long Context": "V4 compressed-entry
// payload" (448 FP8 content channels + 64 BF16 rotary channels, 576 bytes at
// c = 512) and "Quantization scales and bounded tail buffers" (block scale
// metadata).  The scale rule is the OCP Microscaling one, as for the 4-bit
// indexer storage: for a block with largest magnitude amax the byte is
// X + 127 with X = floor(log2 amax) - 8 (8 = E4M3's largest exponent),
// clamped to [-127, 127] (-127 for an all-zero block); each element is
// x / 2^X rounded to the nearest E4M3 value (ties to even, saturating at 448).
// Every dequantized value is a bf16 number, which the attention kernels use:
// they expand the codes exactly into their bf16 tiles.
#include "kernels.h"
#include "lowprec.cuh"

namespace csa {

namespace {

constexpr int kThreads = 256;

// One work item per 32-coordinate content block or 8-coordinate rotary chunk.
__global__ void __launch_bounds__(kThreads) fp8_entry_quantize_kernel(
    const __nv_bfloat16* __restrict__ x, int64_t n, int dim, int rope,
    uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, __nv_bfloat16* __restrict__ rope_out) {
  const int dc = dim - rope, nb = dc / 32, per_row = nb + rope / 8;
  const int64_t it = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (it >= n * per_row) return;
  const int64_t row = it / per_row;
  const int j = (int)(it - row * per_row);
  const __nv_bfloat16* src = x + row * dim;
  if (j >= nb) {   // rotary chunk: kept as it is
    const int c = j - nb;
    *reinterpret_cast<uint4*>(rope_out + row * rope + 8 * c) =
        __ldg(reinterpret_cast<const uint4*>(src + dc + 8 * c));
    return;
  }
  const uint4* p = reinterpret_cast<const uint4*>(src + 32 * j);
  float v[32];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 u = __ldg(p + i);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = unpack_bf16(w[k]);
      v[8 * i + 2 * k] = f.x;
      v[8 * i + 2 * k + 1] = f.y;
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int ef = (int)((__float_as_uint(amax) >> 23) & 0xffu);
  int X = ef == 0 ? -127 : ef - 127 - 8;
  X = X < -127 ? -127 : (X > 127 ? 127 : X);
  const float inv = __uint_as_float((uint32_t)(127 - X) << 23);   // 2^-X, exact
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint32_t word = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) word |= lowprec::e4m3_code(v[4 * i + k] * inv) << (8 * k);
    w[i] = word;
  }
  uint4* dst = reinterpret_cast<uint4*>(codes + row * dc + 32 * j);
  dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
  dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
  scales[row * nb + j] = (uint8_t)(X + 127);
}

}  // namespace

cudaError_t launch_fp8_entry_quantize(const Launch& L, const __nv_bfloat16* x, int64_t n, int dim,
                                      int rope, uint8_t* codes, uint8_t* scales,
                                      __nv_bfloat16* rope_out) {
  const int64_t items = n * ((dim - rope) / 32 + rope / 8);
  if (items == 0) return cudaSuccess;
  L.begin(kKernelQuantize);
  fp8_entry_quantize_kernel<<<(unsigned)((items + kThreads - 1) / kThreads), kThreads, 0, L.stream>>>(
      x, n, dim, rope, codes, scales, rope_out);
  return L.end(kKernelQuantize);
}

}  // namespace csa
