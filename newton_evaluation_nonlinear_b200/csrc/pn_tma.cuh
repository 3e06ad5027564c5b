// pn_tma.cuh -- mbarrier and bulk-copy (TMA) helpers for sm_100a, inline PTX.
//
// Only the untiled global -> shared bulk copy is used
// (cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes), into
// the issuing CTA's own shared memory, never with cluster multicast.  Both
// addresses must be 16-byte aligned and the size a multiple of 16 bytes.
#pragma once

#include "pn_common.cuh"

namespace pn {

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Invalidate a barrier whose operations have all completed, before it is initialised again.
__device__ __forceinline__ void mbar_inval(uint64_t* bar) {
  asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Make barrier initialisation visible to the async (bulk-copy) proxy.
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity to complete.  Gives up
// (returns false) when another CTA has set ctrl->error, or after timeout_ns,
// in which case it sets ctrl->error = PN_ERR_TIMEOUT itself.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned parity, Ctrl* ctrl, long long timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  unsigned spins = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (((++spins) & 31u) == 0u) {
      if (ld_volatile(&ctrl->error)) return false;
      if ((long long)(globaltimer() - t0) > timeout_ns) {
        raise_error(ctrl, (int)PN_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Wait for copies this CTA issued to land, ignoring other CTAs' errors (a CTA
// must not exit with bulk copies into its shared memory in flight).  Bounded
// by timeout_ns; returns false if that ran out.
__device__ __forceinline__ bool mbar_drain(uint64_t* bar, unsigned parity, long long timeout_ns) {
  const unsigned long long t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if ((long long)(globaltimer() - t0) > timeout_ns) return false;
  }
  return true;
}

// Bulk copy of `bytes` (multiple of 16) from global to this CTA's shared
// memory; completion is counted on `bar` (transaction bytes).
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Named barrier over the first `nthreads` threads that also returns, to every one of them, whether
// `v` held on all of them (a warp-aligned instruction: the warp is reconverged first).
__device__ __forceinline__ bool named_barrier_and(unsigned id, unsigned nthreads, bool v) {
  __syncwarp();
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// Named barrier over the first `nthreads` threads (a multiple of 32).
// bar.sync is warp-aligned: every thread of a warp must reach it together, which inline asm does not
// tell the compiler, so the warp is reconverged first (the code before a barrier may have diverged).
__device__ __forceinline__ void named_barrier(unsigned id, unsigned nthreads) {
  __syncwarp();
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

}  // namespace pn
