// pipeline.cuh -- shared-memory barriers and bulk copies (sm_100a PTX), with bounded waits.
//
// Every wait here gives up after kWaitLimitNs of wall-clock time: the caller then records
// NVFP4 error bit 2 (a device-side wait gave up) and leaves its loop, so a lost arrival
// can never hang the GPU.
#pragma once
#include "common.cuh"

namespace nvfp4 {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

// Make initialised barriers visible to the async (TMA) proxy and the other threads.
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
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

// As mbar_try_wait, but a thread whose phase is not complete is suspended until it
// completes or about kSuspendHintNs have passed, instead of returning at once: waiting warps
// then leave the issue slots to the warps that work.
constexpr uint32_t kSuspendHintNs = 1000000;   // 1 ms
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete; false if the limit ran out.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity,
                                          uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait_sleep(bar, parity)) {
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
  return true;
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Wait (one thread) until the global word *p reaches `want` (other CTAs add to it);
// false if *abort was set or the limit ran out (the caller then records the timeout).
__device__ __forceinline__ bool wait_geq(const uint32_t *p, uint32_t want, volatile int *abort,
                                         uint64_t limit_ns = kWaitLimitNs) {
  if (*abort) return false;
  if (ld_acquire_gpu(p) >= want) return true;
  const uint64_t t0 = global_timer_ns();
  while (ld_acquire_gpu(p) < want) {
    if (*abort) return false;
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
  return true;
}

// One-dimensional bulk copy global -> shared, completing `bytes` on the barrier.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes,
                                         uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Bulk copies move 16-byte-aligned runs of a multiple of 16 bytes.  A run of scale rows
// (rows * cols/16 bytes) need not be aligned, so the aligned superset is copied instead:
// it stays inside the expert's own scale block, whose size rows_total * cols/16 is a
// multiple of 16 (rows and cols are multiples of 64).  Returns the bytes issued; the
// wanted data starts `lead` = begin % 16 bytes into dst.
__device__ __forceinline__ uint32_t bulk_g2s_span(void *dst, const uint8_t *block, int64_t begin,
                                                  int64_t len, uint64_t *bar) {
  const int64_t b = begin & ~int64_t(15);
  const int64_t e = (begin + len + 15) & ~int64_t(15);
  bulk_g2s(dst, block + b, (uint32_t)(e - b), bar);
  return (uint32_t)(e - b);
}

__host__ __device__ __forceinline__ uint32_t span_bytes(int64_t len) { return (uint32_t)len + 32; }

// Named barrier among `threads` threads (a multiple of 32) with id 1..15.
__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Record a device-side wait that gave up.
__device__ __forceinline__ void report_timeout(int32_t *flag) {
  if (flag) atomicOr(flag, kFlagWaitTimeout);
}

}  // namespace nvfp4
