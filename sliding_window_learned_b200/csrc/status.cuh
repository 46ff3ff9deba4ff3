// status.cuh -- the device status word and the bound on every device wait.
#pragma once
#include <stdint.h>

namespace attnsink {

// Longest time any single device-side wait may take before the kernel gives
// up, records ATTN_ETIMEOUT and returns (1 s; a healthy wait is microseconds).
constexpr uint64_t kWaitLimitNs = 1000000000ull;

// Must match ATTN_ETIMEOUT and ATTN_ECUDA in include/attnsink.h.
constexpr int kStatusTimeout = -5;
constexpr int kStatusCuda = -3;

// Per-CTA context for bounded waits: a shared abort flag (so one timed-out
// wait stops the whole CTA promptly) and the global status word
// ([0] = code, [1] = location of the first failing wait, [2..3] = the wait
// limit in ns as one 64-bit value, 0 = kWaitLimitNs).
struct WaitCtx {
  volatile int *abort;
  int *status;
  uint64_t limit;   // this launch's wait limit in ns (read once, at the start)
};

// The limit a bounded wait uses: the one set in the status word, else the
// default.  (Waits that drain in-flight copies on the way out keep the
// default, so that a short limit never lets a CTA leave with copies landing.)
__device__ __forceinline__ uint64_t wait_limit_ns(const int *status) {
  const unsigned long long v = *reinterpret_cast<const volatile unsigned long long *>(status + 2);
  return v == 0 ? kWaitLimitNs : static_cast<uint64_t>(v);
}

__device__ __forceinline__ void report_timeout(int *status, int where) {
  if (atomicCAS(status, 0, kStatusTimeout) == 0) atomicExch(status + 1, where);
}

// A kernel that finds its launch unusable (dynamic shared memory not at the
// alignment it declares) records ATTN_ECUDA and returns before any other work.
__device__ __forceinline__ void report_launch_error(int *status, int where) {
  if (atomicCAS(status, 0, kStatusCuda) == 0) atomicExch(status + 1, where);
}

}  // namespace attnsink
