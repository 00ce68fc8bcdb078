// Shared device helpers of the CSA / HCA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/csa.h"

namespace csa {

// ---------------------------------------------------------------------------
// workspace header: the first 256 bytes of every workspace
// ---------------------------------------------------------------------------
struct WsHeader {
  int32_t code;     // 0 = clean, else a DevErr value (first error wins)
  int32_t where;    // query / row index of the first error
  int64_t value;    // offending value (index, page id, ...)
  int32_t pad[60];
};
static_assert(sizeof(WsHeader) == 256, "workspace header is 256 bytes");
constexpr size_t kWsHeader = 256;

enum DevErr : int32_t {
  kErrNone = 0,
  kErrEntryIndex = 1,    // selected entry id outside the cache
  kErrPageId = 2,        // page table entry outside the pool
  kErrEligible = 3,      // eligible entries exceed the workspace layout bound
  kErrWindow = 4,        // window length outside [0, window]
  kErrTimeout = 5,       // a bounded wait on a pipeline barrier gave up
  kErrSelect = 6,        // top-k scratch inconsistent (histogram below k)
};

__device__ __forceinline__ void report(WsHeader* h, int32_t code, int32_t where, int64_t value) {
  if (h == nullptr) return;
  if (atomicCAS(&h->code, 0, code) == 0) {
    h->where = where;
    h->value = value;
  }
}

// ---------------------------------------------------------------------------
// compressed cache addressing (contiguous or paged)
// ---------------------------------------------------------------------------
struct CacheRef {
  const __nv_bfloat16* data;
  int64_t n_rows;
  int64_t seq_stride;
  const int32_t* page_table;
  int32_t page_size;
  int32_t max_pages;
};

// Physical row of entry `e` of sequence `seq`, or -1 (and a report) when the
// row would fall outside the cache.
__device__ __forceinline__ int64_t cache_row(const CacheRef& c, int32_t seq, int64_t e,
                                             WsHeader* err, int32_t where) {
  int64_t row;
  if (c.page_table == nullptr) {
    row = (int64_t)seq * c.seq_stride + e;
    if (e < 0 || (c.seq_stride > 0 && e >= c.seq_stride) || row >= c.n_rows) {
      report(err, kErrEntryIndex, where, e);
      return -1;
    }
  } else {
    int64_t pi = e / c.page_size;
    if (e < 0 || pi >= c.max_pages) {
      report(err, kErrEntryIndex, where, e);
      return -1;
    }
    int32_t page = __ldg(c.page_table + (int64_t)seq * c.max_pages + pi);
    row = (int64_t)page * c.page_size + (e - pi * c.page_size);
    if (page < 0 || row >= c.n_rows) {
      report(err, kErrPageId, where, page);
      return -1;
    }
  }
  return row;
}

// ---------------------------------------------------------------------------
// small PTX wrappers (tensor-core mma.sync, ldmatrix, cp.async)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, bool valid) {
  int sz = valid ? 16 : 0;   // zero-fill when invalid (no global read)
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(sz));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

// streaming 16-byte global load that does not allocate in L1
__device__ __forceinline__ uint4 ld_stream_16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
  __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&u);
  return __bfloat1622float2(v);
}

// Order-preserving map fp32 -> uint32 (larger float -> larger key); -0 and +0
// share one key so that signed zeros tie.
__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t u = __float_as_uint(s);
  if ((u << 1) == 0u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_score(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(u);
}

constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------
// mbarrier + bulk-copy (TMA, non-tensor) helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_cnt(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(bytes)
               : "memory");
}
// Arrive on `bar` once every cp.async issued so far by this thread has landed
// (the arrival is part of the barrier's expected count).
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for the phase of `bar` with the given parity to complete, giving up
// after about `limit_cycles` SM cycles.  Returns false on timeout.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          long long limit_cycles = 2000000000ll) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > limit_cycles) return false;
  return true;
}
// Same, with a suspend-time hint: a waiting thread is parked until the phase
// completes (or the hint, in ns, runs out) instead of polling, so it takes no
// issue slots or shared-memory bandwidth from the threads doing the work.
__device__ __forceinline__ bool mbar_try_wait_susp(uint32_t bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_susp(uint32_t bar, uint32_t parity,
                                               long long limit_cycles = 2000000000ll) {
  if (mbar_try_wait_susp(bar, parity, 100000u)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait_susp(bar, parity, 100000u))
    if (clock64() - t0 > limit_cycles) return false;
  return true;
}
// Same, backing off with nanosleep between polls: for waiters that are not on
// the critical path, so that they leave issue slots to the producer threads.
__device__ __forceinline__ bool mbar_wait_sleep(uint32_t bar, uint32_t parity, unsigned ns = 256,
                                                long long limit_cycles = 2000000000ll) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > limit_cycles) return false;
    __nanosleep(ns);
  }
  return true;
}
// Orders this thread's generic-proxy shared-memory writes before later reads
// by the async proxy (TMA, tcgen05.mma / tcgen05.cp operands).
__device__ __forceinline__ void fence_async_smem_cta() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
// global -> shared bulk copy completing on an mbarrier (both addresses 16-byte
// aligned, size a multiple of 16)
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start before its predecessor ends; pdl_wait() blocks until
// the predecessor has completed and its writes are visible (a no-op in a
// kernel launched normally), pdl_trigger() lets this kernel's own successor
// start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

__device__ __forceinline__ void named_barrier_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(threads) : "memory");
}

}  // namespace csa
