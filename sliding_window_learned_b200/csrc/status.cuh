// status.cuh -- the device status word and the bound on every device wait.
#pragma once
#include <stdint.h>

namespace attnsink {

// Longest time any single device-side wait may take before the kernel gives
// up, records ATTN_ETIMEOUT and returns (1 s; a healthy wait is microseconds).
constexpr uint64_t kWaitLimitNs = 1000000000ull;

// Must match ATTN_ETIMEOUT in include/attnsink.h.
constexpr int kStatusTimeout = -5;

// Per-CTA context for bounded waits: a shared abort flag (so one timed-out
// wait stops the whole CTA promptly) and the global status word
// ([0] = code, [1] = location of the first failing wait).
struct WaitCtx {
  volatile int *abort;
  int *status;
};

__device__ __forceinline__ void report_timeout(int *status, int where) {
  if (atomicCAS(status, 0, kStatusTimeout) == 0) atomicExch(status + 1, where);
}

}  // namespace attnsink
