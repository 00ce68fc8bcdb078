"""fp64 reference of the 4-bit indexer storage format (FP4 values with one
1-byte scale per 32 elements).

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never
imports this module.

Source pages:
  * "DeepSeek-V4" book, Ch.8 "A Cost Model for Long Context", sections "V4
    compressed-entry payload" (the 128-dim indexer key is kept in FP4, half a
    byte per scalar) and "Quantization scales and bounded tail buffers" (one
    1-byte scale factor per 32 elements, +4 bytes per 64-byte key);
  * Ch.6 "Top-k selection and asymptotic scaling" and Ch.8 "Main-attention
    versus indexer arithmetic" (the indexer scan runs on four-bit dot
    products).

Readings taken where the pages are silent:
  Q1  "FP4" is the E2M1 element type (1 sign, 2 exponent, 1 mantissa bit,
      exponent bias 1, no inf / NaN): magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6.
  Q2  the 1-byte scale is a power of two stored as a biased exponent
      (E8M0: byte b means 2^(b-127)), shared by 32 consecutive elements, and
      chosen from the block's largest magnitude as in the OCP Microscaling
      (MX) format: X = floor(log2(amax)) - 2 (2 = E2M1's largest exponent),
      clamped to [-127, 127]; an all-zero block takes X = -127.
  Q3  each element x / 2^X is rounded to the nearest E2M1 value, ties to the
      even code (mantissa bit 0), magnitudes above 6 saturate to 6; the sign
      bit is x's sign bit.
  Q4  byte i of a packed vector holds element 2i in its low nibble and element
      2i+1 in its high nibble; a vector of n elements is n/2 code bytes plus
      n/32 scale bytes (kept in a separate array with the same row order).
  Q5  the quantized indexer applies the ordinary score definition
      I_s = sum_h w_h ReLU(q_h . K_s) to the dequantized queries and keys;
      w stays fp32.
"""
from __future__ import annotations

import numpy as np

BLOCK = 32          # elements sharing one scale byte (Ch.8, scale factors)
E2M1_EMAX = 2       # exponent of E2M1's largest value, 6 = 1.5 * 2^2


def e2m1_value(code):
    """Value of a 4-bit E2M1 code (reading Q1), from its bit fields:
    sign = bit 3, exponent e = bits 2..1, mantissa f = bit 0;
    e = 0 is subnormal (f * 0.5), else 2^(e-1) * (1 + f/2)."""
    code = np.asarray(code, dtype=np.int64)
    s = (code >> 3) & 1
    e = (code >> 1) & 3
    f = code & 1
    mag = np.where(e == 0, 0.5 * f, np.ldexp(1.0 + 0.5 * f, e - 1))
    return np.where(s == 1, -mag, mag)


def e2m1_encode(y):
    """Nearest E2M1 code of each y (reading Q3): brute force over the eight
    magnitudes, ties to the even code, saturation at 6 (the nearest
    magnitude of anything above 6 is 6 itself)."""
    y = np.asarray(y, dtype=np.float64)
    mags = e2m1_value(np.arange(8))                          # [8], increasing
    dist = np.abs(np.abs(y)[..., None] - mags)              # [..., 8]
    best = dist.min(axis=-1, keepdims=True)
    tied = dist == best
    # among the nearest magnitudes prefer an even code; there is always
    # exactly one even code among at most two neighbours
    even = tied & (np.arange(8) % 2 == 0)
    pick = np.where(even.any(axis=-1), np.argmax(even, axis=-1), np.argmax(tied, axis=-1))
    sign = np.signbit(y).astype(np.int64)
    return (pick + 8 * sign).astype(np.uint8)


def mxfp4_scale_exponent(block):
    """Shared exponent X of one block of 32 values (reading Q2)."""
    amax = float(np.max(np.abs(np.asarray(block, dtype=np.float64))))
    if amax == 0.0:
        return -127
    _, e = np.frexp(amax)            # amax = f * 2^e, f in [0.5, 1)
    return int(min(max(e - 1 - E2M1_EMAX, -127), 127))


def mxfp4_quantize(x):
    """Quantize rows of x ([..., n], n a multiple of 32) to packed E2M1 codes
    [..., n/2] (uint8, reading Q4) and E8M0 scale bytes [..., n/32]: per block
    of 32 the shared exponent of reading Q2, then reading Q3 per element."""
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[-1]
    assert n % BLOCK == 0, "the vector length must be a multiple of 32"
    blocks = x.reshape(-1, BLOCK)                            # one row per scale block
    amax = np.abs(blocks).max(axis=1)
    _, e = np.frexp(amax)                                    # amax = f * 2^e, f in [0.5, 1)
    X = np.where(amax == 0.0, -127, np.clip(e - 1 - E2M1_EMAX, -127, 127)).astype(np.int64)
    codes = e2m1_encode(blocks / np.ldexp(1.0, X)[:, None]).reshape(-1, n)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    scales = (X + 127).astype(np.uint8)
    return packed.reshape(x.shape[:-1] + (n // 2,)), scales.reshape(x.shape[:-1] + (n // BLOCK,))


def mxfp4_dequantize(packed, scales):
    """Values of packed codes [..., n/2] with scale bytes [..., n/32], fp64."""
    packed = np.asarray(packed, dtype=np.uint8)
    scales = np.asarray(scales, dtype=np.int64)
    n = packed.shape[-1] * 2
    codes = np.empty(packed.shape[:-1] + (n,), dtype=np.int64)
    codes[..., 0::2] = packed & 0xF
    codes[..., 1::2] = packed >> 4
    vals = e2m1_value(codes)
    factor = np.repeat(np.ldexp(1.0, scales - 127), BLOCK, axis=-1)
    return vals * factor


def indexer_scores_mxfp4(q_packed, q_scales, w, k_packed, k_scales):
    """Indexer scores over 4-bit queries and keys (reading Q5): the score
    definition of Ch.6 "The lightning indexer" on the dequantized values.
    q_packed [H_I, c_I/2], q_scales [H_I, c_I/32], w [H_I],
    k_packed [n, c_I/2], k_scales [n, c_I/32]; returns [n]."""
    q = mxfp4_dequantize(q_packed, q_scales)
    K = mxfp4_dequantize(k_packed, k_scales)
    w = np.asarray(w, dtype=np.float64)
    return np.maximum(K @ q.T, 0.0) @ w
