// common.cuh -- device helpers shared by the EPLB kernels (sm_100a).
//
// Hand-written PTX for the Blackwell bulk-copy engine: 1-D cp.async.bulk
// global->shared copies that complete on a shared-memory mbarrier
// (transaction-count based), plus bounded waits.  No copy here uses cluster
// multicast; every source address is this GPU's own global memory.
#pragma once

#include <cstdint>

#include "../../include/eplb.h"

namespace eplb {

// Upper bound of any in-kernel wait, in nanoseconds of %globaltimer.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

// Makes initialised mbarriers visible to the async (bulk-copy) proxy.
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for phase `parity` of `bar`; false if it did not complete within
// kWaitLimitNs (the caller reports EPLB_ERR_TIMEOUT and drains).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  for (;;) {
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
}

// 1-D bulk copy global -> this CTA's shared memory, completing `bytes`
// transactions on `bar`.  dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes,
                                         uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Same, with an L2 evict-first policy for data read exactly once.
__device__ __forceinline__ void bulk_g2s_stream(void *dst, const void *src, uint32_t bytes,
                                                uint64_t *bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ void report(int32_t *status, int32_t code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

// x mod d for 0 <= x < 2^31 and 1 <= d < 2^31 with m = floor((2^32-1)/d):
// q = floor(x*m / 2^32) undershoots floor(x/d) by at most 1 (the deficit
// x*(2^32/d - m)/2^32 < 2x/2^32 < 1), so one conditional subtraction fixes
// the remainder.  Multiply-high division after Granlund & Montgomery,
// "Division by invariant integers using multiplication", PLDI 1994.
// Shared-memory access by 32-bit shared-window address: one multiply-add
// per address, no generic-pointer arithmetic.
__device__ __forceinline__ void red_shared_inc(uint32_t addr) {
  asm volatile("red.shared.add.u32 [%0], 1;" ::"r"(addr));
}
__device__ __forceinline__ int32_t ld_shared_s16(uint32_t addr) {
  int32_t v;
  asm volatile("ld.shared.s16 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

// Programmatic dependent launch.  Every kernel of the library is launched
// with programmatic stream serialisation: at its start it lets the next
// kernel of the stream be scheduled (pdl_trigger) and then waits until the
// previous grid of the stream has finished and its memory is visible
// (pdl_wait) before it touches global memory, so launch latency overlaps
// the previous kernel's tail while stream order still holds for every read
// and write.  Both are no-ops for a kernel launched without the attribute.
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ uint32_t mod_magic(uint32_t x, uint32_t d, uint32_t m) {
  uint32_t q = __umulhi(x, m);
  uint32_t r = x - q * d;
  return r >= d ? r - d : r;
}
__device__ __forceinline__ uint32_t div_magic(uint32_t x, uint32_t d, uint32_t m) {
  uint32_t q = __umulhi(x, m);
  return (x - q * d) >= d ? q + 1 : q;
}

}  // namespace eplb
