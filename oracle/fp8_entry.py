"""fp64 reference of the mixed-precision compressed-entry storage: FP8 content
coordinates with one scale byte per 32, the rotary coordinates kept in bf16.

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never
imports this module.

Source pages:
  * "DeepSeek-V4" book, Ch.8 "A Cost Model for Long Context", section "V4
    compressed-entry payload": each shared KV entry keeps its non-rotary
    content channels in FP8 (1 byte each) and its last 64 rotary channels in
    BF16 (2 bytes each), 448 + 128 = 576 bytes at c = 512; section
    "Quantization scales and bounded tail buffers": block-quantized FP8
    tensors carry scale metadata beside the packed values;
  * Ch.7 "Partial RoPE and output de-rotation" (the rotary slice is the last
    64 coordinates).

Readings taken where the pages are silent:
  F1  "FP8" is E4M3 without infinities (1 sign, 4 exponent bits with bias 7,
      3 mantissa bits; exponent field 0 is subnormal; the all-ones pattern is
      NaN): largest magnitude 448, smallest 2^-9.
  F2  the content coordinates are quantized in blocks of 32 sharing one
      power-of-two scale byte, as in the OCP Microscaling format (the same rule
      as the 4-bit indexer storage): X = floor(log2 amax) - 8 (8 = E4M3's
      largest exponent), clamped to [-127, 127], -127 for an all-zero block;
      byte X + 127.
  F3  each x / 2^X is rounded to the nearest E4M3 value, ties to the even
      code, saturating at 448; the sign bit is x's sign bit.
  F4  an entry of d coordinates with r rotary ones is stored as d - r code
      bytes, (d - r) / 32 scale bytes and r bf16 values, in three arrays with
      the same row order; the dequantized entry is the concatenation of the
      scaled content and the rotary part.
  F5  attention over such entries is the ordinary shared-KV attention over the
      dequantized entries (every dequantized value is a bf16 number, so the
      dequantized cache is exactly a bf16 cache).
"""
from __future__ import annotations

import numpy as np

BLOCK = 32            # content coordinates sharing one scale byte
E4M3_EMAX = 8         # exponent of E4M3's largest value, 448 = 1.75 * 2^8
E4M3_MAX_CODE = 0x7E  # 448; 0x7F is NaN


def e4m3_value(code):
    """Value of an 8-bit E4M3 code (reading F1) from its bit fields:
    sign = bit 7, exponent E = bits 6..3, mantissa M = bits 2..0;
    E = 0: M * 2^-9, else (1 + M/8) * 2^(E-7); 0x7F / 0xFF are NaN."""
    code = np.asarray(code, dtype=np.int64)
    s = (code >> 7) & 1
    E = (code >> 3) & 15
    M = code & 7
    mag = np.where(E == 0, M * 2.0 ** -9, np.ldexp(1.0 + M / 8.0, E - 7))
    mag = np.where((code & 0x7F) == 0x7F, np.nan, mag)
    return np.where(s == 1, -mag, mag)


def e4m3_encode(y):
    """Nearest E4M3 code of each y (reading F3): of the two finite magnitudes
    that bracket |y| (clamped to 448: saturation) the nearer one, ties to the
    even code."""
    y = np.asarray(y, dtype=np.float64)
    mags = e4m3_value(np.arange(E4M3_MAX_CODE + 1))         # increasing, 0 .. 448
    a = np.minimum(np.abs(y), mags[-1])
    hi = np.clip(np.searchsorted(mags, a, side="left"), 0, E4M3_MAX_CODE)   # mags[hi] >= a
    lo = np.clip(hi - 1, 0, E4M3_MAX_CODE)
    d_lo, d_hi = a - mags[lo], mags[hi] - a
    pick = np.where(d_lo < d_hi, lo, np.where(d_hi < d_lo, hi, np.where(lo % 2 == 0, lo, hi)))
    sign = np.signbit(y).astype(np.int64)
    return (pick + 128 * sign).astype(np.uint8)


def mxfp8_scale_exponent(block):
    """Shared exponent X of one block of 32 values (reading F2)."""
    amax = float(np.max(np.abs(np.asarray(block, dtype=np.float64))))
    if amax == 0.0:
        return -127
    _, e = np.frexp(amax)            # amax = f * 2^e, f in [0.5, 1)
    return int(min(max(e - 1 - E4M3_EMAX, -127), 127))


def mxfp8_quantize(x):
    """Rows of x ([..., n], n a multiple of 32) -> E4M3 codes [..., n] and
    scale bytes [..., n/32] (uint8): per block the exponent of reading F2,
    then reading F3 per element."""
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[-1]
    assert n % BLOCK == 0, "the vector length must be a multiple of 32"
    blocks = x.reshape(-1, BLOCK)
    amax = np.abs(blocks).max(axis=1)
    _, e = np.frexp(amax)
    X = np.where(amax == 0.0, -127, np.clip(e - 1 - E4M3_EMAX, -127, 127)).astype(np.int64)
    codes = e4m3_encode(blocks / np.ldexp(1.0, X)[:, None])
    return codes.reshape(x.shape), (X + 127).astype(np.uint8).reshape(x.shape[:-1] + (n // BLOCK,))


def mxfp8_dequantize(codes, scales):
    """Values of E4M3 codes [..., n] with scale bytes [..., n/32], fp64."""
    scales = np.asarray(scales, dtype=np.int64)
    return e4m3_value(codes) * np.repeat(np.ldexp(1.0, scales - 127), BLOCK, axis=-1)


def entry_quantize(x, rope_dims):
    """Entries x [..., d] -> (codes [..., d - r], scales [..., (d - r)/32],
    rope [..., r]) under reading F4; the rotary part is returned as given
    (the caller's bf16 values)."""
    x = np.asarray(x, dtype=np.float64)
    dc = x.shape[-1] - rope_dims
    codes, scales = mxfp8_quantize(x[..., :dc])
    return codes, scales, x[..., dc:].copy()


def entry_dequantize(codes, scales, rope):
    """The entries [..., d] that the stored parts represent (reading F4)."""
    return np.concatenate([mxfp8_dequantize(codes, scales), np.asarray(rope, dtype=np.float64)],
                          axis=-1)
