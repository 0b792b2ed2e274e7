// Bulk asynchronous global -> shared copies (the untiled TMA path) completed
// on a shared-memory mbarrier, with a bounded wait.
//
// Rules the callers keep: source and destination 16-byte aligned, sizes a
// multiple of 16 bytes, at most 2^20 - 1 bytes expected per barrier phase. No
// cluster multicast is used; each CTA copies only into its own shared memory.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace gs {

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// One-thread initialisation of an mbarrier expecting one arrival per phase,
// made visible to the asynchronous proxy before any copy references it.
__device__ __forceinline__ void mbar_init(uint64_t* bar) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(bar)) : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// The one arrival of the phase, announcing `bytes` of copies that will complete on it.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

// Copies `bytes` from global `src` to shared `dst`, completing on `bar`.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Starts bringing `bytes` at `src` into L2 (same alignment rules as a copy;
// nothing to wait for: a later copy of the same bytes finds them in L2).
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Waits for phase `parity` of `bar` to complete, polling at most `max_polls`
// times; returns false if it gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int max_polls) {
  for (int k = 0; k < max_polls; ++k) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}

// After a bounded wait has given up: keeps waiting for the phase with a
// backoff (1 us sleeps, about `max_us` microseconds in all), so that the CTA
// does not retire - and its shared memory is not handed to another CTA -
// while copies into it may still be in flight. Returns true if the phase
// completed. The copies only fail to land when the memory system has faulted;
// if even this wait gives up, the CTA retires with the copies outstanding and
// the recorded error makes the launch's results unusable.
__device__ __forceinline__ bool mbar_drain(uint64_t* bar, uint32_t parity, int max_us) {
  for (int k = 0; k < max_us; ++k) {
    if (mbar_wait(bar, parity, 1)) return true;
    __nanosleep(1000);
  }
  return false;
}

}  // namespace gs
