// Device helpers shared by the decode-attention kernels (sm_100a): mbarrier
// and 1-D bulk-copy wrappers (cp.async.bulk, never with cluster multicast),
// bounded waits, mma.sync / ldmatrix wrappers and small warp reductions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kvq_internal.cuh"

namespace kvq {
namespace {

// floor(a / b) for 0 <= a < 2^50 and b > 0, given rb = 1 / b rounded to double.
// The 64-bit integer division is a long serial subroutine (the partition math
// of a decode launch took microseconds with it); the double estimate is
// within one of the quotient and is then corrected exactly in integers.
__device__ __forceinline__ int64_t div_floor(int64_t a, int64_t b, double rb) {
  int64_t q = (int64_t)((double)a * rb);
  while (q > 0 && q * b > a) --q;
  while ((q + 1) * b <= a) ++q;
  return q;
}
__device__ __forceinline__ double recip(int64_t b) { return __drcp_rn((double)b); }

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
// The same test, but a thread whose phase is not complete may sleep up to
// `ns` nanoseconds (it resumes when the phase completes), instead of spinning
// on issue slots the compute warps need.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* b, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}
// Bounded wait: false if the phase did not complete within `limit` SM cycles
// or the CTA is already aborting.  The default bound, kWaitCycles, is about
// 1 s at the B200's top clock; the decode launches take theirs from the launch
// arguments (a test may shorten it, see kvq_debug_set_wait_test).  Waits for
// copies in flight before a CTA exits always use the default bound.
constexpr long long kWaitCycles = kWaitCyclesDefault;
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, volatile int* abort_flag,
                                          long long limit = kWaitCycles) {
  if (mbar_try_wait(b, parity)) return true;
  const long long t0 = clock64();
  const uint32_t ns = limit < 40000ll ? 0u : 20000u;   // a short bound polls instead of sleeping
  for (;;) {
    if (mbar_try_wait_sleep(b, parity, ns)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > limit) return false;
  }
}
// Waits (bounded by the default limit) for a phase whose copy is in flight,
// so that no bulk copy still writes this CTA's shared memory when it exits.
__device__ __forceinline__ void mbar_drain(uint64_t* b, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(b, parity) && clock64() - t0 < kWaitCycles) {
  }
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
// Records first .. first + cnt - 1 of a row (cnt <= 16) into shared memory,
// in steps so that a paged cache's page-id loads are in flight while the
// producer waits for a free stage:
//   record_pages  issues the loads of the ids of the pages the records touch;
//   pages_valid   (after the wait) whether all of them are in the pool;
//   copy_records  arms `bar` and issues one copy per page.
// (Paged caches only; a contiguous stage is one copy issued directly.)
struct RecordPages {
  int32_t ids[16];
  int nr, p0;
};
// Page sizes are powers of two (page_shift = log2 of records per page), so the
// page arithmetic is shifts and masks on 32-bit record indices.
__device__ __forceinline__ void record_pages(const Geom& gm, int row, int64_t first, int cnt, RecordPages& pg) {
  const int f = (int)first, sh = gm.page_shift;
  pg.p0 = f >> sh;
  pg.nr = ((f + cnt - 1) >> sh) - pg.p0 + 1;
  const int32_t* tab = gm.page_table + (int64_t)row * gm.pages_per_row + pg.p0;
  pg.ids[0] = __ldg(tab);
  if (pg.nr > 1) {
#pragma unroll
    for (int i = 1; i < 16; ++i) pg.ids[i] = i < pg.nr ? __ldg(tab + i) : 0;
  }
}
__device__ __forceinline__ bool pages_valid(const Geom& gm, const RecordPages& pg) {
  if (pg.nr == 1) return pg.ids[0] >= 0 && pg.ids[0] < gm.num_pages;
  bool ok = true;
#pragma unroll
  for (int i = 0; i < 16; ++i)
    if (i < pg.nr && (pg.ids[i] < 0 || pg.ids[i] >= gm.num_pages)) ok = false;
  return ok;
}
__device__ __forceinline__ void copy_records(const Geom& gm, int row, int64_t first, int cnt, int rec_bytes,
                                             const RecordPages& pg, unsigned char* dst, uint64_t* bar) {
  mbar_expect_tx(bar, (uint32_t)cnt * rec_bytes);
  const int f = (int)first, sh = gm.page_shift, mask = (1 << sh) - 1;
  if (pg.nr == 1) {
    bulk_g2s(dst, gm.records + (((int64_t)pg.ids[0] << sh) | (f & mask)) * rec_bytes, (uint32_t)cnt * rec_bytes,
             bar);
    return;
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    if (i < pg.nr) {
      const int pgi = pg.p0 + i;
      const int g0 = max(f, pgi << sh), g1 = min(f + cnt, (pgi + 1) << sh);
      bulk_g2s(dst + (int64_t)(g0 - f) * rec_bytes,
               gm.records + (((int64_t)pg.ids[i] << sh) | (g0 & mask)) * rec_bytes, (uint32_t)(g1 - g0) * rec_bytes,
               bar);
    }
  }
}

__device__ __forceinline__ void mma_bf16_16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t* r, const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(row_addr)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t* r, const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(row_addr)));
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t* r, const void* row_addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];\n"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(smem_u32(row_addr)));
}
// two floats -> packed pair in the input's 16-bit format
__device__ __forceinline__ uint32_t pack2_in16(float lo, float hi, int dtype) {
  if (dtype == KVQ_FP16) return h2_as_u32(__floats2half2_rn(lo, hi));
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&b);
}
__device__ __forceinline__ float2 unpack2_in16(uint32_t w, int dtype) {
  if (dtype == KVQ_FP16) return __half22float2(u32_as_h2(w));
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
// named barrier 1 over the N consumer threads of a warp-specialized CTA
template <int N>
__device__ __forceinline__ void named_bar_sync() {
  asm volatile("bar.sync 1, %0;\n" ::"n"(N) : "memory");
}
__device__ __forceinline__ uint4 lds128(const void* p) { return *reinterpret_cast<const uint4*>(p); }
__device__ __forceinline__ uint32_t in16x2_to_h2(uint32_t w, int dtype) {
  if (dtype == KVQ_FP16) return w;
  return h2_as_u32(__floats2half2_rn(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u)));
}
__device__ __forceinline__ float quad_max(float x) {
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1));
  return fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 2));
}
__device__ __forceinline__ float quad_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  return x + __shfl_xor_sync(0xffffffffu, x, 2);
}

}  // namespace
}  // namespace kvq
