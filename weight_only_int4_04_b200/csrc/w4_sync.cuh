// mbarrier, bulk-copy and timer helpers (inline PTX, sm_100a). Every wait is bounded: after
// kWaitLimitNs of wall time it records W4_ERR_TIMEOUT in the library's device error word and
// sets a CTA-wide abort flag so that the remaining waits of the CTA give up at once; the
// kernel then runs to its end on whatever data it has, and the host sees the error through
// w4_device_error(). No wait can hang the GPU.
//
// Abort path: a CTA must not exit while bulk copies it issued can still write its shared
// memory, nor free tensor memory that an MMA it issued may still write. So the stages a ring
// issued are waited for (mbar_drain: bounded, but deaf to the abort flag) before the CTA
// exits -- by the issuing thread itself in the GEMV kernels; in the tcgen05 GEMM, after the
// CTA's final barrier and only when the abort flag is up, by one thread that also waits for
// the MMA issuer's last commit before the tensor memory is freed (drain code inside the
// GEMM's producer and MMA branches measured 4-5% slower prefill, although it never ran).
#pragma once

#include <stdint.h>

#include "w4_internal.cuh"

namespace w4i {

constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s: far above any legitimate wait

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Makes the initialized barriers visible to the async proxy (bulk copies, tensor core).
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// try_wait with a suspend-time hint: the waiting thread sleeps until the phase completes or
// about `ns` nanoseconds pass, instead of spinning through issue slots.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity, uint32_t ns) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
      : "memory");
  return done != 0;
}

// Bounded wait for the phase with the given parity to complete. Returns false if it gave up
// (timeout here or an abort raised elsewhere in the CTA). A caller must never wait for a
// phase more than one ahead of the barrier's last completed phase (parity would alias).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                          int32_t *err, uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t n = 0;; ++n) {
    // The hint lets the hardware suspend the thread until the phase completes (it wakes on
    // completion, not on a timer), so a waiter takes no issue slots and resumes at once.
    const uint32_t hint = limit_ns < 1000000u ? static_cast<uint32_t>(limit_ns) + 1u : 1000000u;
    if (mbar_try_wait_sleep(bar, parity, hint)) return true;
    if (n >= 32) __nanosleep(256);  // only if the suspend keeps returning early
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      if (err) atomicExch(err, static_cast<int32_t>(W4_ERR_TIMEOUT));
      return false;
    }
  }
}

// Wait for a phase that copies or MMAs this thread issued will complete, whatever the abort
// flag says (their writes must land before the CTA exits or frees tensor memory). Bounded by
// kWaitLimitNs like every other wait; gives up with W4_ERR_TIMEOUT recorded.
__device__ __forceinline__ void mbar_drain(uint64_t *bar, uint32_t parity, int32_t *err) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t n = 0;; ++n) {
    if (mbar_try_wait_sleep(bar, parity, 1000000u)) return;
    if (n >= 32) __nanosleep(256);
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      if (err) atomicExch(err, static_cast<int32_t>(W4_ERR_TIMEOUT));
      return;
    }
  }
}

// One-dimensional bulk copy global -> shared, completing `bytes` on the mbarrier.
// Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_copy_g2s(void *dst_smem, const void *src_gmem, uint32_t bytes,
                                              uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst_smem)),
      "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void named_barrier_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Programmatic dependent launch. A kernel launched with programmatic stream serialization
// may start while the previous kernel of its stream is still running; grid_dependency_wait
// blocks the calling thread until that kernel has completed and its memory writes are
// visible (it returns at once when there is no such dependency).
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Allows the next kernel of the stream (if launched with programmatic serialization) to be
// scheduled once every CTA of this grid has executed this or exited.
__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace w4i
