// Bulk global -> shared copies completed on an mbarrier, with bounded waits,
// for the CUDA-core kernel's key staging.  Plain `cp.async.bulk` (no tensor
// map, no cluster multicast): the source is this GPU's own memory.
#pragma once

#include <cstdint>

namespace va {
namespace bulk {

constexpr unsigned long long kTimeoutNs = 1000000000ull;  // 1 s per wait

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      "selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}
// Wait for phase `parity` of a local barrier for at most kTimeoutNs; false
// if it did not complete in time.
__device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity) {
  const unsigned long long t0 = global_ns();
  for (;;) {
#pragma unroll 1
    for (int k = 0; k < 32; ++k)
      if (mbar_try(bar, parity)) return true;
    if (global_ns() - t0 > kTimeoutNs) return false;
  }
}
__device__ __forceinline__ bool mbar_wait(uint64_t* barp, uint32_t parity) {
  const uint32_t bar = smem_u32(barp);
  if (mbar_try(bar, parity)) return true;
  return mbar_wait_slow(bar, parity);
}
// One arrival that also announces `bytes` of copies still to land.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
               ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
// Orders this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (bulk copy) accesses of the same bytes.
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Makes an initialised mbarrier visible to the async proxy.
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// Copy `bytes` (a multiple of 16; both addresses 16-byte aligned) from
// global to this CTA's shared memory; completion counted on `bar`.
__device__ __forceinline__ void copy_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// After an expired wait: give copies already in flight time to land before
// the CTA exits (bounded busy wait, 200 us).
__device__ __noinline__ void settle() {
  const unsigned long long t0 = global_ns();
  while (global_ns() - t0 < 200000ull) { }
}

}  // namespace bulk
}  // namespace va
