// Decode-time cache maintenance: one new token per sequence.
//
// DeepSeek-V4 book, Ch.5 "Decode-time cache state" (the compressed cache grows
// by one entry every m decode steps; bounded tail buffers hold the sliding
// window, the b-branch rows of the just-completed block and the tokens of the
// unfinished block) and Ch.8 "Quantization scales and bounded tail buffers".
//
// One CTA per sequence, one thread per 8 coordinates.  The token's rows go to
// the window ring (slot t mod W) and to the block buffers (row t mod m; in
// overlap mode its b-branch rows to the buffer of block parity (t / m) & 1).
// When the token completes block i = t / m, the bulk compressor's pooling
// routine turns the block (and block i-1's b-branch rows) into entry i of the
// compressed cache, so the entry has the same bits as from csa_compress_kv.
// Each thread reads back only the coordinates it wrote, so no barrier is needed.
#include "pooling.cuh"

namespace csa {

namespace {

__global__ void cache_append_kernel(CacheAppendArgs a) {
  const int b = blockIdx.x;
  const int v = threadIdx.x;
  if (v >= (a.dim >> 3)) return;
  const int dim = a.dim, m = a.m, c0 = v * 8;
  const int64_t t = __ldg(a.pos + b);
  if (t < 0) {
    if (v == 0) report(a.err, kErrEntryIndex, b, t);
    return;
  }
  const int j = (int)(t % m);
  const int64_t i = t / m;
  const int64_t src = (int64_t)b * dim + c0;
  const uint4 ca = *reinterpret_cast<const uint4*>(a.Ca + src);
  const uint4 za = *reinterpret_cast<const uint4*>(a.Za + src);
  if (a.window > 0)
    *reinterpret_cast<uint4*>(a.win + ((int64_t)b * a.window + t % a.window) * dim + c0) = ca;
  *reinterpret_cast<uint4*>(a.blk_c + ((int64_t)b * m + j) * dim + c0) = ca;
  *reinterpret_cast<uint4*>(a.blk_z + ((int64_t)b * m + j) * dim + c0) = za;
  if (a.overlap) {
    const uint4 cb = *reinterpret_cast<const uint4*>((a.Cb ? a.Cb : a.Ca) + src);
    const uint4 zb = *reinterpret_cast<const uint4*>((a.Zb ? a.Zb : a.Za) + src);
    const int64_t rb = (((int64_t)b * 2 + (i & 1)) * m + j) * dim + c0;
    *reinterpret_cast<uint4*>(a.bb_c + rb) = cb;
    *reinterpret_cast<uint4*>(a.bb_z + rb) = zb;
  }
  if (j != m - 1) return;
  // block i is complete: entry i
  pooling::Acc8 A;
  pooling::init(A);
  pooling::pool_rows<false>(A, a.blk_c, a.blk_z, a.bias, (int64_t)b * m, m, dim, c0);
  if (a.overlap && i > 0)
    pooling::pool_rows<false>(A, a.bb_c, a.bb_z, a.bias ? a.bias + (int64_t)m * dim : nullptr,
                              ((int64_t)b * 2 + ((i - 1) & 1)) * m, m, dim, c0);
  if (i >= a.max_entries) {
    if (v == 0) report(a.err, kErrEntryIndex, b, i);
    return;
  }
  const int64_t row = cache_row(a.cache, b, i, a.err, b);
  if (row < 0) return;
  *reinterpret_cast<uint4*>(const_cast<__nv_bfloat16*>(a.cache.data) + row * dim + c0) = pooling::finish(A);
}

}  // namespace

cudaError_t launch_cache_append(const Launch& L, const CacheAppendArgs& a) {
  if (a.B == 0) return cudaSuccess;
  const int threads = ((a.dim >> 3) + 31) / 32 * 32;
  L.begin(kKernelCompress);
  cache_append_kernel<<<(unsigned)a.B, threads, 0, L.stream>>>(a);
  return L.end(kKernelCompress);
}

}  // namespace csa
