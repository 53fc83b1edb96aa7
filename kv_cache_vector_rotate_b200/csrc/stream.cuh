// Device helpers shared by the streaming kernels (logits, values): shared
// memory addresses, bounded mbarrier waits, bulk copies, mma.sync wrappers.
#pragma once

#include "tq_internal.cuh"

namespace tqd {

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

constexpr long long kWaitCycles = 2000000000LL;   // ~1 s: a bounded mbarrier wait gives up after this

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}
// A plain arrival (no transaction bytes).
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}
// One test of the phase of the given parity.
__device__ __forceinline__ bool mbar_try(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(done) : "r"(smem_addr(bar)), "r"(parity) : "memory");
  return done != 0;
}
// One non-blocking test of the phase of the given parity.
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(done) : "r"(smem_addr(bar)), "r"(parity) : "memory");
  return done != 0;
}
// Waits for the phase of the given parity; false after kWaitCycles.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try(bar, parity)) return true;      // the usual case: no clock read
  const long long t0 = clock64();
  while (true) {
    if (mbar_try(bar, parity)) return true;
    if (clock64() - t0 > kWaitCycles) return false;
  }
}
// One test of the phase with a suspend-time hint: the thread may sleep up to
// `ns` nanoseconds in the test (waking when the phase completes) instead of
// spinning, so waiting warps leave the issue slots to working ones.
__device__ __forceinline__ bool mbar_try_sleep(uint64_t* bar, uint32_t parity, uint32_t ns) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(done) : "r"(smem_addr(bar)), "r"(parity), "r"(ns) : "memory");
  return done != 0;
}
// mbar_wait for waits that may be long: between tests the warp sleeps
// (32 ns, doubling to `max_ns`) and leaves the issue slots to working warps;
// false after kWaitCycles.
__device__ __forceinline__ bool mbar_wait_backoff(uint64_t* bar, uint32_t parity, uint32_t max_ns = 256u) {
  if (mbar_test(bar, parity)) return true;
  const long long t0 = clock64();
  uint32_t ns = 32u;
  while (true) {
    __nanosleep(ns);
    if (mbar_test(bar, parity)) return true;
    if (clock64() - t0 > kWaitCycles) return false;
    ns = ns < max_ns ? 2u * ns : max_ns;
  }
}
// mbar_wait with sleeping tests; false after kWaitCycles.
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t* bar, uint32_t parity) {
  if (mbar_try_sleep(bar, parity, 20000u)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_sleep(bar, parity, 20000u)) return true;
    if (clock64() - t0 > kWaitCycles) return false;
  }
}
// Bulk copy (no multicast) of `bytes` global -> shared, completing on `bar`;
// both addresses 16-byte aligned, bytes a multiple of 16, with an L2
// eviction-priority policy.
__device__ __forceinline__ void bulk_copy(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar,
                                          uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
      ::"r"(dst), "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(pol) : "memory");
}
// Prefetch of `bytes` global bytes into L2 (no data to the SM); the address
// 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
// Bulk copy global -> shared with the default L2 policy (data that other
// CTAs read again, such as constant tables).
__device__ __forceinline__ void bulk_copy_plain(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(dst), "l"(src), "r"(bytes), "r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ void mma_f16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint2 b) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b.x), "r"(b.y));
}

// Four 8 x 8 fp16 matrices from shared memory, transposed (lane i gives the
// address of row i % 8 of matrix i / 8).
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                              uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr) : "memory");
}

}  // namespace tqd
