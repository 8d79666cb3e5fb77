// Bounded waits on shared-memory barriers and small helpers shared by the
// forward and backward kernels.  Every wait gives up after a time limit (the
// globaltimer) or a poll count, records BSA_ERR_DEVICE_TIMEOUT in the status
// word, raises the CTA's abort flag and returns false, so a kernel that cannot
// make progress ends instead of hanging the GPU.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "../../include/bsa.h"
#include "sm100_ptx.cuh"

namespace bsa {

constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;
constexpr uint32_t kMaxSpin = 1u << 24;
constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;
constexpr uint32_t kWaitSleepNs = 20000;  // upper bound on one sleep inside a barrier wait

// Device status word of this translation unit: 0, or the first error a kernel
// recorded (BSA_ERR_DEVICE_TIMEOUT).  Each .cu file that includes this header has
// its own copy and reads and clears it from its host code.
static __device__ int g_bsa_status;

// ------------------------------------------------------------ bounded waits
__device__ __forceinline__ bool wait_spin(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t timeout_ns, bool honor_abort) {
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    // sleeping in the barrier instead of spinning leaves issue slots to the
    // warps that share this SM sub-partition
    if (ptx::mbar_try_wait_sleep(bar, parity, kWaitSleepNs)) return true;
    if ((it & 15u) == 0) {
      if (honor_abort && *abort_flag) return false;
      if (ptx::globaltimer_ns() - t0 > timeout_ns || it > kMaxSpin) {
        *abort_flag = 1;
        atomicCAS(&g_bsa_status, 0, static_cast<int>(BSA_ERR_DEVICE_TIMEOUT));
        return false;
      }
    }
  }
}

// The slow path, out of line.  kRegion tells apart the copies called from warps with
// different register budgets (setmaxnreg): one function may be called only from code
// compiled to one budget, so each such region gets its own instantiation.
template <int kRegion>
__device__ __noinline__ bool wait_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                       uint64_t timeout_ns, bool honor_abort) {
  return wait_spin(bar, parity, abort_flag, timeout_ns, honor_abort);
}

// Whole-warp wait; the result is warp-uniform.
template <int kRegion = 0>
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t timeout_ns) {
  bool ok = ptx::mbar_try_wait(bar, parity);
  if (__all_sync(0xffffffffu, ok)) return true;
  ok = wait_slow<kRegion>(bar, parity, abort_flag, timeout_ns, true);
  return __all_sync(0xffffffffu, ok);
}

template <int kRegion = 0>
__device__ __forceinline__ void wait_force(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                           uint64_t timeout_ns) {
  if (!ptx::mbar_try_wait(bar, parity)) wait_slow<kRegion>(bar, parity, abort_flag, timeout_ns, false);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ------------------------------------------------------------ roles
// Single-thread wait (the TMA and MMA roles run on one elected lane).
template <int kRegion = 0>
__device__ __forceinline__ bool wait_one(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         uint64_t timeout_ns) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  return wait_slow<kRegion>(bar, parity, abort_flag, timeout_ns, true);
}

}  // namespace bsa
