// common.cuh - device status word, bounded barrier waits, small helpers.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace lora {

// Device-side status: bit 0 = a bounded wait gave up.  `g_status_info`
// records the first failure: {block, thread, site code, parity}.  (The
// library is one translation unit, so the definitions live here.)
__device__ unsigned int g_status = 0;
__device__ unsigned int g_status_info[4] = {0, 0, 0, 0};

enum WaitSite : uint32_t {
  SITE_FULL = 1, SITE_EMPTY = 2, SITE_VFULL = 3, SITE_VEMPTY = 4, SITE_ACCFULL = 5,
  SITE_ACCEMPTY = 6, SITE_TFULL = 7, SITE_STFULL = 8, SITE_DRAIN = 9, SITE_SELFTEST = 10,
  SITE_TXMSG = 11, SITE_TXFLAG = 12,
};

// Wait for the phase of `bar` with the given parity to complete.  Spins on
// try_wait; every 64 misses it looks at the CTA's abort flag and at the
// global timer, and gives up (returning false) once `limit_ns` has passed or
// another role of the CTA has already given up.  On the first give-up it
// raises the CTA abort flag and records the failure in the status word.
// `cluster_scope` makes the wait an acquire at cluster scope, for barriers
// that other CTAs of the cluster arrive on.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                             uint64_t limit_ns, uint32_t site, bool cluster_scope = false) {
  auto probe = [&]() { return cluster_scope ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity); };
  if (probe()) return true;
  const uint64_t t0 = global_timer_ns();
  uint32_t spins = 0;
  while (true) {
    if (probe()) return true;
    if ((++spins & 63u) == 0u) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > limit_ns) {
        *abort_flag = 1;
        if (atomicOr(&g_status, 1u) == 0u) {
          g_status_info[0] = blockIdx.x + (blockIdx.y << 16);
          g_status_info[1] = threadIdx.x;
          g_status_info[2] = site;
          g_status_info[3] = parity;
        }
        __threadfence();
        return false;
      }
    }
  }
}

// Wait until the global word `p` reads `want` (acquire at GPU scope), with
// the same limit and give-up behaviour as wait_bounded.
__device__ __forceinline__ bool wait_word_bounded(const uint32_t* p, uint32_t want, volatile int* abort_flag,
                                                  uint64_t limit_ns, uint32_t site) {
  if (ld_acquire_gpu(p) == want) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    __nanosleep(64);
    if (ld_acquire_gpu(p) == want) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      if (atomicOr(&g_status, 1u) == 0u) {
        g_status_info[0] = blockIdx.x + (blockIdx.y << 16);
        g_status_info[1] = threadIdx.x;
        g_status_info[2] = site;
        g_status_info[3] = want;
      }
      __threadfence();
      return false;
    }
  }
}

// Warp-converged form for warps that go on to run .sync.aligned tcgen05
// instructions: lane 0 polls, the result is broadcast, and __syncwarp
// orders the other lanes after lane 0's observation of the barrier.
__device__ __forceinline__ bool warp_wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                                  uint64_t limit_ns, uint32_t site, bool cluster_scope = false) {
  int ok = 1;
  if ((threadIdx.x & 31u) == 0u) ok = wait_bounded(bar, parity, abort_flag, limit_ns, site, cluster_scope) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

// Sleep-wait until `ns` nanoseconds have passed (used on the abort path to
// let copies already in flight land before shared memory is released).
__device__ __forceinline__ void settle_ns(uint64_t ns) {
  const uint64_t t0 = global_timer_ns();
  while (global_timer_ns() - t0 < ns) __nanosleep(1000);
}

__device__ __forceinline__ int imin(int a, int b) { return a < b ? a : b; }

}  // namespace lora
