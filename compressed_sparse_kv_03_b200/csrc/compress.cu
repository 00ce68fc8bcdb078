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
#include "pooling.cuh"

namespace csa {

namespace {

using pooling::Acc8;
constexpr int kThreads = 256;

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
  pooling::init(A);
  // a branch: block i with (C_a, Z_a + bias[0])
  pooling::pool_rows<true>(A, Ca, Za, bias, (int64_t)m * i, m, dim, c0);
  // b branch: block i-1 with (C_b, Z_b + bias[1]); block 0 has none
  if (overlap && i > 0)
    pooling::pool_rows<true>(A, Cb, Zb, bias ? bias + (int64_t)m * dim : nullptr, (int64_t)m * (i - 1), m,
                             dim, c0);
  *reinterpret_cast<uint4*>(out + i * dim + c0) = pooling::finish(A);
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
  prefer_max_shared(compress_kernel);
  compress_kernel<<<blocks, kThreads, 0, L.stream>>>(Ca, Za, Cb ? Cb : Ca, Zb ? Zb : Za, bias, S,
                                                     dim, m, overlap, out);
  return L.end(kKernelCompress);
}

}  // namespace csa
