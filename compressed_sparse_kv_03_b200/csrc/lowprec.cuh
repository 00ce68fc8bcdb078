// E4M3 and E8M0 conversions of the mixed-precision entry storage (FP8
// content coordinates with a power-of-two scale byte per 32, rotary part in
// bf16): DeepSeek-V4 book, Ch.8 "A Cost Model for Long Context", "V4
// compressed-entry payload".  E4M3 here is the variant without infinities:
// sign, 4 exponent bits with bias 7 (field 0 subnormal), 3 mantissa bits,
// largest value 448.
#pragma once

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

}  // namespace lowprec
}  // namespace csa
