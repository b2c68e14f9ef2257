// eqlin_wait.cuh -- bounded mbarrier waits shared by the tensor-core kernels.
//
// Every wait polls at most `limit` times and at most kWaitCycles SM cycles.
// A wait that runs out records where it gave up in the handle's error record
// (first writer wins) and returns false; the kernel then raises its CTA-wide
// abort flag, drains its own in-flight copies and MMAs, frees TMEM and
// returns.  A wait that returns because another role raised the abort flag
// records nothing.
//
// Error record (device, 4 x int32, zeroed at handle creation and by
// eqlin_get_error):
//   [0] status: DEV_OK, or DEV_TIMEOUT
//   [1] site of the first wait that ran out: (kernel << 8) | (role << 4) | barrier
//   [2] that CTA's blockIdx.x | (stage or tile counter << 12)
//   [3] polls made | (milliseconds waited, at the maximum SM clock, << 20)
#pragma once

#include "eqlin_internal.cuh"
#include "eqlin_ptx.cuh"

namespace eqlin {
namespace waits {

using namespace ptx;

// kernels
enum : uint32_t { K_APPLY = 1, K_DW = 2, K_DWS = 3 };

__device__ __forceinline__ uint32_t site(uint32_t kernel, uint32_t role, uint32_t barrier) {
  return (kernel << 8) | (role << 4) | barrier;
}

__device__ __forceinline__ void record_timeout(int* err, uint32_t where, uint32_t iter, uint32_t polls,
                                               uint64_t cycles) {
  if (atomicCAS(err + 1, 0, (int)where) == 0) {
    err[2] = (int)((blockIdx.x & 0xFFFu) | (iter << 12));
    const uint64_t ms = cycles / kCyclesPerMs;
    err[3] = (int)((polls > 0xFFFFFu ? 0xFFFFFu : polls) | ((ms > 0xFFFu ? 0xFFFu : (uint32_t)ms) << 20));
  }
  atomicCAS(err, DEV_OK, DEV_TIMEOUT);
}

// Wait for the phase with the given parity; false if the wait ran out
// (recorded) or another role raised the abort flag (not recorded).
__device__ __forceinline__ bool bwait(uint64_t* bar, uint32_t parity, uint32_t limit, volatile int* abort_flag,
                                      int* err, uint32_t where, uint32_t iter) {
  if (mbar_test_wait(bar, parity)) return true;     // already complete: no suspension
  const uint64_t t0 = cycles_now();
  uint64_t t = t0;
  uint32_t i = 0;
  for (; i < limit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 15u) == 15u) {
      if (*abort_flag) return false;
      t = cycles_now();
      if (t - t0 > kWaitCycles) break;
    }
  }
  record_timeout(err, where, iter, i, t - t0);
  return false;
}

// Wait until the global flag reads `want` (GPU-scope acquire), bounded and
// recorded as the mbarrier waits are.
__device__ __forceinline__ bool flag_wait(const int* flag, int want, uint32_t limit, volatile int* abort_flag,
                                          int* err, uint32_t where, uint32_t iter) {
  const uint64_t t0 = cycles_now();
  uint64_t t = t0;
  uint32_t i = 0;
  for (; i < limit; ++i) {
    if (ld_acquire_gpu(flag) == want) return true;
    __nanosleep(32);
    if ((i & 15u) == 15u) {
      if (*abort_flag) return false;
      t = cycles_now();
      if (t - t0 > kWaitCycles) break;
    }
  }
  record_timeout(err, where, iter, i, t - t0);
  return false;
}

// Lane 0 waits; the warp then agrees on the outcome (and is ordered after the
// wait), so no lane leaves a loop that holds warp-synchronous operations.
__device__ __forceinline__ bool wwait(uint64_t* bar, uint32_t parity, uint32_t limit, volatile int* abort_flag,
                                      int lane, int* err, uint32_t where, uint32_t iter) {
  int ok = 0;
  if (lane == 0) ok = bwait(bar, parity, limit, abort_flag, err, where, iter) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

// Every lane waits (each acquires the phase, as a reader of TMA-written data
// must); the warp agrees on the outcome.
__device__ __forceinline__ bool wwait_all(uint64_t* bar, uint32_t parity, uint32_t limit, volatile int* abort_flag,
                                          int* err, uint32_t where, uint32_t iter) {
  return __all_sync(0xffffffffu, bwait(bar, parity, limit, abort_flag, err, where, iter));
}

__device__ __forceinline__ void raise_abort(volatile int* abort_flag, int* err) {
  *abort_flag = 1;
  atomicCAS(err, DEV_OK, DEV_TIMEOUT);
}

}  // namespace waits
}  // namespace eqlin
