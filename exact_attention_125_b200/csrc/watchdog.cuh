// watchdog.cuh - bounded mbarrier waits.
//
// Every wait in the library's kernels goes through these helpers. A wait that
// has not completed after `limit_ns` nanoseconds of %globaltimer sets the
// CTA's abort flag (shared memory) and ORs kDevErrTimeout into the global
// error word, and returns false; every other wait in the CTA then returns
// false at its next poll, so all roles fall through to the teardown (drain own
// copies, free tensor memory, exit) instead of spinning forever.
#pragma once
#include <cstdint>

#include "sm100.cuh"

namespace attn {

constexpr unsigned int kDevErrTimeout = 1u;

struct Watchdog {
  volatile uint32_t* abort;  // CTA-wide abort flag in shared memory
  unsigned int* err;         // device-global error word
  uint64_t limit_ns;
};

__device__ __forceinline__ bool timed_out(uint64_t t0, const Watchdog& w) {
  if (global_timer_ns() - t0 <= w.limit_ns) return false;
  *w.abort = 1u;
  atomicOr(w.err, kDevErrTimeout);
  return true;
}

// Wait by the MMA-issuing thread for a softmax hand-off: spins on test_wait
// (which never suspends the thread) and checks the abort flag and the time
// limit every 64 polls. try_wait may suspend a thread for a while after the
// phase completes; on the MMA thread that latency sits on every step's
// critical path (measured: the spinning issuer wakes ~100-150 cycles sooner
// after a long wait).
__device__ __forceinline__ bool wait_spin(uint32_t bar, uint32_t parity, const Watchdog& w) {
  uint64_t t0 = 0;
  for (uint32_t it = 0;; ++it) {
    if (mbar_test_wait(bar, parity)) return true;
    if ((it & 63) == 63) {
      if (t0 == 0) t0 = global_timer_ns();
      if (*w.abort) return false;
      if (timed_out(t0, w)) return false;
    }
  }
}

// Wait by a single thread (TMA producer, MMA issuer).
__device__ __forceinline__ bool wait_one(uint32_t bar, uint32_t parity, const Watchdog& w) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*w.abort) return false;
    if (timed_out(t0, w)) return false;
  }
}

// Wait by a whole warp that then issues warp-collective tcgen05 instructions:
// every lane polls, and the outcome is made warp-uniform.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const Watchdog& w) {
  if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
  const bool leader = lane_id() == 0;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    const bool done = mbar_try_wait(bar, parity);
    if (__all_sync(0xffffffffu, done)) return true;
    uint32_t stop = 0;
    if (leader) stop = (*w.abort != 0u) || timed_out(t0, w);
    if (__shfl_sync(0xffffffffu, stop, 0)) return false;
  }
}

// Teardown wait for a thread's own in-flight asynchronous work (TMA copies,
// tcgen05 MMAs): ignores the abort flag, still bounded by limit_ns.
__device__ __forceinline__ bool drain_wait(uint32_t bar, uint32_t parity, const Watchdog& w) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > w.limit_ns) {
      atomicOr(w.err, kDevErrTimeout);
      return false;
    }
  }
}

}  // namespace attn
