// common.cuh -- device helpers shared by the EPLB kernels (sm_100a): shared
// addresses, the status word, multiply-high division by per-divisor magic
// numbers, 32-bit shared-address access, programmatic dependent launch.
#pragma once

#include <cstdint>

#include "../../include/eplb.h"

namespace eplb {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void report(int32_t *status, int32_t code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

// Checking build (-DEPLB_CHECKS): EPLB_IN(cond, status) states an index
// bound the kernel relies on (a shared-memory row or slot, an output
// position derived from data); when it does not hold, the access it guards
// is skipped and EPLB_ERR_INTERNAL goes to the call's status word.  In the
// normal build it is the constant true and the guard compiles away.
#ifdef EPLB_CHECKS
__device__ __forceinline__ bool check_in(bool cond, int32_t *status) {
  if (!cond) report(status, EPLB_ERR_INTERNAL);
  return cond;
}
#define EPLB_IN(cond, status) (::eplb::check_in((cond), (status)))
#else
#define EPLB_IN(cond, status) true
#endif

// Shared-memory access by 32-bit shared-window address: one multiply-add
// per address, no generic-pointer arithmetic.
__device__ __forceinline__ void red_shared_inc(uint32_t addr) {
  asm volatile("red.shared.add.u32 [%0], 1;" ::"r"(addr));
}
__device__ __forceinline__ uint64_t ld_shared_u64(uint32_t addr) {
  uint64_t v;
  asm volatile("ld.shared.u64 %0, [%1];" : "=l"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ void ld_shared_u64x2(uint32_t addr, uint64_t &x, uint64_t &y) {
  asm volatile("ld.shared.v2.u64 {%0, %1}, [%2];" : "=l"(x), "=l"(y) : "r"(addr));
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

// Brings the 128-byte line holding p into L2.  It reads nothing into the
// thread and L2 is the point of coherence for global memory, so it may be
// issued before pdl_wait, even on data the previous grid is still writing.
__device__ __forceinline__ void prefetch_l2(const void *p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// x mod d for 0 <= x < 2^31 and 1 <= d < 2^31 with m = floor((2^32-1)/d):
// q = floor(x*m / 2^32) undershoots floor(x/d) by at most 1 (the deficit
// x*(2^32/d - m)/2^32 < 2x/2^32 < 1), so one conditional subtraction fixes
// the remainder.  Multiply-high division after Granlund & Montgomery,
// "Division by invariant integers using multiplication", PLDI 1994.
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
