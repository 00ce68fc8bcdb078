// Block-wide helpers of the exact top-k selection kernels (NT threads, a
// multiple of 32 up to 1024): an exclusive scan, the histogram bin that holds
// the k-th largest key, and the two bitmap steps that end every selection
// (lowest-index ties, then an ascending compaction of the selected entries).
#pragma once

#include "common.cuh"

namespace csa {
namespace sel {

// Block-wide exclusive scan of one int per thread; returns this thread's
// prefix and sets `total`.  Every thread must call it; warp_sums holds 32 ints.
template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_sums, int& total) {
  constexpr int kWarps = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int s = lane < kWarps ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    warp_sums[lane] = s;   // inclusive prefix of warp totals
  }
  __syncthreads();
  total = warp_sums[kWarps - 1];
  const int base = warp ? warp_sums[warp - 1] : 0;
  __syncthreads();   // warp_sums is reused by the next scan
  return base + x - v;
}

// Bin holding the `need`-th largest element of a histogram of `nbins` bins
// (nbins a multiple of NT): sets *bin and *above (elements in higher bins)
// and returns true.  If the histogram holds fewer than `need` elements
// (inconsistent scratch) it returns false with *bin = 0 and *above = 0, so that
// every later index stays in range.  Every thread must call it.
template <int NT>
__device__ __forceinline__ bool find_bin(const int* hist, int nbins, int need, int* warp_sums,
                                         uint32_t* s_bin, int* s_above, int* s_ok) {
  if (threadIdx.x == 0) {
    *s_bin = 0u;
    *s_above = 0;
    *s_ok = 0;
  }
  const int per = nbins / NT;
  // thread i owns ranks [i*per, (i+1)*per) counted from the top bin down
  int c = 0;
  for (int r = 0; r < per; ++r) c += hist[nbins - 1 - (threadIdx.x * per + r)];
  int tot;
  int before = block_exclusive_scan<NT>(c, warp_sums, tot);   // syncs order the defaults first
  for (int r = 0; r < per; ++r) {
    const int b = nbins - 1 - (threadIdx.x * per + r);
    const int h = hist[b];
    if (before < need && before + h >= need) {
      *s_bin = (uint32_t)b;
      *s_above = before;
      *s_ok = 1;
    }
    before += h;
  }
  __syncthreads();
  return *s_ok != 0;
}

// Ties at the k-th key: the first `need` set bits of tie[0 .. W) in index
// order join sel[].  Every thread must call it.
template <int NT>
__device__ __forceinline__ void take_lowest_ties(uint32_t* sel, const uint32_t* tie, int W,
                                                 int need, int* warp_sums) {
  const int wpt = (W + NT - 1) / NT;
  const int w0 = threadIdx.x * wpt, w1 = min(W, w0 + wpt);
  int c = 0;
  for (int w = w0; w < w1; ++w) c += __popc(tie[w]);
  int tot;
  int before = block_exclusive_scan<NT>(c, warp_sums, tot);
  for (int w = w0; w < w1; ++w) {
    uint32_t x = tie[w];
    const int pc = __popc(x);
    int take = need - before;
    take = take < 0 ? 0 : (take > pc ? pc : take);
    uint32_t kept = 0;
    for (int i = 0; i < take; ++i) {
      const uint32_t low = x & (0u - x);
      kept |= low;
      x ^= low;
    }
    sel[w] |= kept;
    before += pc;
  }
  __syncthreads();
}

// Ascending compaction of the selection bitmap sel[0 .. W): the i-th set bit
// (in index order) is written to idx[i] for i < k, and on_sel(i, j) is called
// for it (j the entry index).  Every thread must call it.
template <int NT, class F>
__device__ __forceinline__ void compact_ascending(const uint32_t* sel, int W, int k, int32_t* idx,
                                                  int* warp_sums, F on_sel) {
  const int wpt = (W + NT - 1) / NT;
  const int w0 = threadIdx.x * wpt, w1 = min(W, w0 + wpt);
  int c = 0;
  for (int w = w0; w < w1; ++w) c += __popc(sel[w]);
  int tot;
  int o = block_exclusive_scan<NT>(c, warp_sums, tot);
  for (int w = w0; w < w1; ++w) {
    uint32_t x = sel[w];
    while (x) {
      const int b = __ffs(x) - 1;
      x &= x - 1;
      if (o < k) {
        const int64_t j = (int64_t)w * 32 + b;
        idx[o] = (int32_t)j;
        on_sel(o, j);
      }
      ++o;
    }
  }
}

}  // namespace sel
}  // namespace csa
