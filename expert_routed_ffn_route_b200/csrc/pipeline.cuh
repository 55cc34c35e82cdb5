// Device-side building blocks for asynchronous tile movement on sm_100a: mbarriers,
// one-dimensional bulk copies (TMA engine, no multicast), bounded waits and programmatic
// dependent launch control.
#pragma once

#include "common.cuh"

namespace moe {

// A wait that has not completed after this many SM clock cycles (about 2 s at 1.9 GHz)
// gives up and reports DEV_TIMEOUT instead of hanging the GPU.
constexpr long long kWaitCycles = 4000000000LL;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
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

// Waits for the phase of `bar` with the given parity to complete; false on timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) return false;
  }
  return true;
}

// Non-blocking test of the phase with the given parity (mbarrier.test_wait).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait that polls with the non-blocking test. For barriers completed by other
// threads' arrivals, a thread suspended inside try_wait was measured on B200 to notice the
// completion microseconds late; a polling thread notices it at once.
__device__ __forceinline__ bool mbar_wait_poll(uint64_t* bar, uint32_t parity) {
  if (mbar_test_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_test_wait(bar, parity)) {
    if (clock64() - t0 > kWaitCycles) return false;
  }
  return true;
}

// Bulk copy global -> shared (this CTA), completion counted on `bar` in bytes.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Orders this thread's generic-proxy shared-memory writes before later async-proxy reads
// (TMA stores, tensor-core operand fetches) of the same memory.
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Programmatic dependent launch: wait for the preceding kernel's results (no-op when the
// kernel was launched without the programmatic serialisation attribute) ...
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// ... and allow the next kernel in the stream to start its prologue.
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------------ grid barrier

// Grid-wide barrier on one 32-bit word whose low 31 bits are zero between barriers (the
// workspace starts zeroed). Every CTA adds to the word exactly once per barrier; CTA 0 adds
// 2^31 - (grid - 1) and the others 1, so the top bit flips exactly when the last CTA
// arrives, in whatever order they come, and the low bits are zero again afterwards. A CTA is
// through once it sees the top bit differ from the value it found on arrival. A CTA that
// gave up waiting still left its arrival behind, so a late arrival completes its own
// barrier and never leaks into the next one; the grid size may change from call to call.
__device__ __forceinline__ void fence_acq_rel_gpu() {
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

// Arrival: a release (this CTA's writes, ordered before it by the CTA barrier the caller
// has passed, become visible to every CTA that sees the arrival).
__device__ __forceinline__ uint32_t gbar_arrive(uint32_t* bar) {
  const uint32_t add = (blockIdx.x == 0) ? (0x80000000u - (gridDim.x - 1)) : 1u;
  fence_acq_rel_gpu();
  return atomicAdd(bar, add);
}

// Waits (boundedly) until the barrier `arrived` (the value gbar_arrive returned) completes.
__device__ __forceinline__ bool gbar_wait(const uint32_t* bar, uint32_t arrived) {
  const long long t0 = clock64();
  while (true) {
    uint32_t now;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(now) : "l"(bar) : "memory");
    if ((now ^ arrived) & 0x80000000u) break;
    if (clock64() - t0 > kWaitCycles) return false;
    __nanosleep(32);
  }
  return true;
}

// ------------------------------------------------------------------ failure injection

// Test hook: while the workspace's hold word (test_ctl[0]) is nonzero, the kernels that
// check it wait for it to return to zero, which nothing does during the call, so the wait
// runs out after test_ctl[1] clock cycles (kWaitCycles when that is zero) and reports
// DEV_TIMEOUT, exactly as a wait on a peer that never arrives would. Returns false on that
// timeout; true at once when the hold word is zero (the normal case: one load).
__device__ __forceinline__ bool test_hold_wait(const int32_t* test_ctl) {
  if (!test_ctl) return true;
  if (__ldcg(test_ctl) == 0) return true;
  const int32_t budget = __ldcg(test_ctl + 1);
  const long long limit = budget > 0 ? (long long)budget : kWaitCycles;
  const long long t0 = clock64();
  while (*(volatile const int32_t*)test_ctl != 0) {
    if (clock64() - t0 > limit) return false;
    __nanosleep(64);
  }
  return true;
}

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// CTA barrier `id` of `threads` threads that warps may reach from different places in the
// code (the non-aligned form of the barrier); whole, converged warps only.
__device__ __forceinline__ void bar_sync_any(int id, int threads) {
  asm volatile("barrier.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Arrives at named barrier `id` (of `threads` threads) without waiting; whole warps only.
__device__ __forceinline__ void named_bar_arrive(int id, int threads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(threads) : "memory");
}


}  // namespace moe
