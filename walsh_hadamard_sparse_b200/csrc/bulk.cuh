// mbarrier and untiled bulk-copy (TMA engine) helpers for kernels that stream
// contiguous rows into a shared-memory ring. Every wait is bounded.
#pragma once

#include <stdint.h>

namespace qwha {
namespace bulk {

constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint32_t saddr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Make the initialised barriers visible to the async proxy (the copy engine).
__device__ __forceinline__ void fence_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

// Order this thread's earlier generic-proxy accesses of shared memory before
// later async-proxy ones (a copy that overwrites a slot other threads read).
__device__ __forceinline__ void fence_proxy() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ bool try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase of the given parity to complete; false once limit_ns
// have passed since the first unsuccessful poll. A limit of 0 gives up at
// once without polling (how a test makes a wait run out deterministically).
__device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity, uint64_t limit_ns = kWaitNs) {
  if (limit_ns == 0) return false;
  if (try_wait(bar, parity)) return true;
  const uint64_t t0 = now_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (try_wait(bar, parity)) return true;
    if (now_ns() - t0 > limit_ns) return false;
  }
}

// Copy `bytes` (a multiple of 16; both addresses 16-byte aligned) from global
// memory into this CTA's shared memory, completing on `bar` (whose expected
// transaction count the caller has raised). No multicast.
__device__ __forceinline__ void copy(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Arrive on `bar` announcing `bytes` of copies that will complete on it, then
// copy `bytes` (a multiple of 16; both addresses 16-byte aligned) from global
// memory into this CTA's shared memory. No multicast.
__device__ __forceinline__ void load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Copy `bytes` (a multiple of 16; both addresses 16-byte aligned) from this
// CTA's shared memory to global memory, in the current bulk group.
__device__ __forceinline__ void store(void *dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// This thread's committed stores have read their shared-memory sources (the
// writes themselves complete before the grid does).
__device__ __forceinline__ void wait_stores_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

}  // namespace bulk
}  // namespace qwha
