// E4M3 and E8M0 conversions of the mixed-precision entry storage (FP8
// content coordinates with a power-of-two scale byte per 32, rotary part in
// bf16): DeepSeek-V4 book, Ch.8 "A Cost Model for Long Context", "V4
// compressed-entry payload".  E4M3 here is the variant without infinities:
// sign, 4 exponent bits with bias 7 (field 0 subnormal), 3 mantissa bits,
// largest value 448.
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"

namespace csa {
namespace lowprec {

// 2^(b - 127) for a scale byte b (b = 0: 2^-127, a subnormal)
__device__ __forceinline__ float e8m0_to_float(uint32_t b) {
  return b ? __uint_as_float(b << 23) : __uint_as_float(0x00400000u);
}

// Value of an E4M3 code, exactly (every E4M3 number is an fp32 number).
__device__ __forceinline__ float e4m3_to_float(uint32_t c) {
  const uint32_t E = (c >> 3) & 15u, M = c & 7u;
  const float v = E ? __uint_as_float(((E + 120u) << 23) | (M << 20))   // (1 + M/8) 2^(E-7)
                    : (float)M * 0.001953125f;                            // M 2^-9
  return (c & 0x80u) ? -v : v;
}

// Two E4M3 codes (bits 0-7 and 8-15 of `two`) times fs, rounded to a bf16
// pair (low half = the first code): the hardware pair conversion to f16 is
// exact, so is the fp32 product with a power of two, and the bf16 rounding
// equals that of e4m3_to_float(c) * fs.
__device__ __forceinline__ uint32_t e4m3x2_scaled_bf16x2(uint32_t two, float fs) {
  uint32_t h2;
  asm("{\n .reg .b16 t;\n cvt.u16.u32 t, %1;\n cvt.rn.f16x2.e4m3x2 %0, t;\n}\n" : "=r"(h2) : "r"(two));
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
  return pack_bf16(f.x * fs, f.y * fs);
}

// Nearest E4M3 code of y, ties to the even code, saturating at 448; the sign
// bit is y's.  In the binade of floor(log2 |y|) (at least -6, the subnormal
// range) the representable values are integers m times 2^(e-3), so the code
// is the rounded m (round-half-even) above the binade's first code.
__device__ __forceinline__ uint32_t e4m3_code(float y) {
  const float a = fabsf(y);
  uint32_t c;
  if (a >= 448.f) {
    c = 0x7Eu;
  } else {
    int e = (int)((__float_as_uint(a) >> 23) & 0xffu) - 127;
    e = e < -6 ? -6 : e;
    const float m = rintf(a * __uint_as_float((uint32_t)(130 - e) << 23));   // a * 2^(3-e)
    c = (uint32_t)(((e + 7) << 3) + (int)m - 8);
  }
  return c | ((__float_as_uint(y) >> 31) << 7);
}


// Nearest E2M1 code of y (4-bit indexer format): magnitudes 0, 0.5, 1, 1.5,
// 2, 3, 4, 6, ties to the even code, saturating at 6; the sign bit is y's.
__device__ __forceinline__ uint32_t e2m1_code(float y) {
  const float a = fabsf(y);
  // nearest magnitude, ties to the even code (0, 1, 1.5 -> 2, 2 -> 4, 4 -> 6)
  uint32_t c = a <= 0.25f ? 0u
             : a < 0.75f  ? 1u
             : a <= 1.25f ? 2u
             : a < 1.75f  ? 3u
             : a <= 2.5f  ? 4u
             : a < 3.5f   ? 5u
             : a <= 5.0f  ? 6u
                          : 7u;
  return c | ((__float_as_uint(y) >> 31) << 3);
}

// One 32-element block of the 4-bit indexer format (E2M1 codes, one
// power-of-two scale byte): its four code words (nibble j of word i = element
// 8i + j) and its scale byte.  The standalone quantizer, the scorer's query
// prologue and the selection's own scoring all use this, so their codes are
// identical.
__device__ __forceinline__ uint32_t quantize_block(const __nv_bfloat16* __restrict__ src,
                                                   uint32_t (&out)[4]) {
  const uint4* p = reinterpret_cast<const uint4*>(src);
  float v[32];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 u = __ldg(p + i);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = unpack_bf16(w[j]);
      v[8 * i + 2 * j] = f.x;
      v[8 * i + 2 * j + 1] = f.y;
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  // floor(log2 amax) from the exponent field; subnormal or zero amax clamps
  // to the smallest scale
  const int ef = (int)((__float_as_uint(amax) >> 23) & 0xffu);
  int X = ef == 0 ? -127 : ef - 127 - 2;
  X = X < -127 ? -127 : (X > 127 ? 127 : X);
  const float inv = __uint_as_float((uint32_t)(127 - X) << 23);   // 2^-X, exact
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) word |= e2m1_code(v[8 * i + j] * inv) << (4 * j);
    out[i] = word;
  }
  return (uint32_t)(X + 127);
}


// Value of an E2M1 code (sign bit 3, exponent bits 2-1 with bias 1, mantissa
// bit 0): exactly one of +-{0, 0.5, 1, 1.5, 2, 3, 4, 6}.
__device__ __forceinline__ float e2m1_to_float(uint32_t c) {
  const uint32_t E = (c >> 1) & 3u, M = c & 1u;
  const float v = E ? __uint_as_float(((E + 126u) << 23) | (M << 22))   // (1 + M/2) 2^(E-1)
                    : 0.5f * (float)M;
  return (c & 8u) ? -v : v;
}

}  // namespace lowprec
}  // namespace csa
