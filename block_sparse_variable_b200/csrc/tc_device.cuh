// tc_device.cuh -- bounded mbarrier waits shared by the tcgen05 kernels.
#pragma once

#include <stdint.h>

#include "bsa_internal.h"
#include "sm100.cuh"

namespace bsa {

constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s: any legitimate wait is far shorter

static __device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Longest single hardware suspension of a waiting thread (ns).  A thread
// whose barrier never completes (another role aborted) notices the abort flag
// within this time.
constexpr uint32_t kSuspendNs = 200000;

// Bounded wait: the thread sleeps in the barrier (no polling loop competing
// for issue slots with the math warps) and gives up after kWaitNs of wall
// time (raising the abort flag and BSA_FLAG_TIMEOUT), or as soon as another
// role has aborted.
static __device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int *abort,
                                         uint32_t *status) {
  if (sm100::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (;;) {
    if (sm100::mbar_try_wait_sleep(bar, parity, kSuspendNs)) return true;
    if (*abort) return false;
    if (global_ns() - t0 > kWaitNs) {
      *abort = 1;
      atomicOr(status + kStFlags, BSA_FLAG_TIMEOUT);
      return false;
    }
  }
}

// Producers run ahead of their consumers; the same wait serves them.
static __device__ __forceinline__ bool wait_bar_lazy(uint32_t bar, uint32_t parity,
                                              volatile int *abort, uint32_t *status) {
  return wait_bar(bar, parity, abort, status);
}

static __device__ __forceinline__ bool wait_warp_lazy(uint32_t bar, uint32_t parity,
                                               volatile int *abort, uint32_t *status) {
  const bool r = wait_bar(bar, parity, abort, status);
  return __all_sync(0xffffffffu, r);
}

// the same, agreed by the whole warp (tcgen05 .sync.aligned ops follow)
static __device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, volatile int *abort,
                                          uint32_t *status) {
  const bool r = wait_bar(bar, parity, abort, status);
  return __all_sync(0xffffffffu, r);
}

// drain wait on the abort path: bounded, result ignored
static __device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = global_ns();
  while (!sm100::mbar_try_wait(bar, parity) && global_ns() - t0 < kWaitNs) {
  }
}

}  // namespace bsa
