// decode_noalloc.cu -- attn_sink_decode_noalloc: the split-KV decode with its
// workspace in a fixed-size array of device memory that belongs to the
// library image, so the call itself allocates nothing.
//
// For callers that must not allocate device memory during a decode step: for
// example a serving engine that reserves (nearly) all of HBM up front for its
// KV cache and forbids allocations by the libraries it calls, or a runtime
// whose own allocator owns every device byte.  In such a process a
// stream-ordered allocation can fail or take time and memory the caller has
// not budgeted, so attn_sink_decode's pooled workspace is not an option.
//
// The array lives in this translation unit only, so with lazy module loading a
// process that never calls this entry point does not pay for it.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/attnsink.h"
#include "api_internal.h"
#include "kernels.h"

namespace attnsink {
namespace {

// Largest workspace this entry point can use (plan + partial LSEs + partial
// outputs): 48 MiB.  Held on every device that loads this module, until exit.
constexpr size_t kScratchBytes = static_cast<size_t>(48) << 20;
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices];

// Device address of the scratch array on the current device.  In host code
// `g_decode_scratch` names a host-side shadow, not device memory, so the
// address is looked up once per device (with that device current).
int scratch_address(void **out) {
  int dev;
  int rc = current_device(&dev);
  if (rc) return rc;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return fail_cuda(e, "cudaGetSymbolAddress(decode scratch)");
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return ATTN_OK;
}

}  // namespace
}  // namespace attnsink

using namespace attnsink;

extern "C" int attn_sink_decode_noalloc(const attn_tensor *q, const attn_tensor *kcache,
                                        const attn_tensor *vcache, const attn_tensor *seqlens,
                                        const attn_tensor *sinks, int32_t window, float scale,
                                        attn_tensor *out, void *stream) {
  clear_error();
  DecodeArgs a;
  bool empty;
  int rc = prep_decode(q, kcache, vcache, seqlens, sinks, window, scale, 0, out, &a, &empty);
  if (rc || empty) return rc;
  const size_t need = decode_workspace_bytes(a);
  if (need > kScratchBytes)
    return fail(ATTN_EUNSUPPORTED,
                "decode needs %zu bytes of workspace; the no-allocation entry point has %zu "
                "(B * ceil(min(Smax, window) / chunk) splits * Hq * (D + 1) * 4 bytes)",
                need, kScratchBytes);
  if ((rc = status_ptr(&a.status))) return rc;
  void *ws = nullptr;
  if ((rc = scratch_address(&ws))) return rc;
  // Nothing in the scratch array needs to start at zero: the planner kernel
  // rewrites the split table and resets the work counter on every call, and
  // every partial that the combine reads is written by the split kernel first.
  const cudaError_t e = launch_decode(a, ws, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? ATTN_OK : fail_cuda(e, "attn_sink_decode_noalloc launch");
}
