// api_internal.h -- host helpers shared by the C-ABI translation units.
#pragma once
#include "../../include/attnsink.h"
#include "kernels.h"

namespace attnsink {

// Clears the calling thread's attn_sink_last_error() message.
void clear_error();
// Records a one-line message for attn_sink_last_error() and returns `code`.
int fail(int code, const char *fmt, ...);
// Maps a CUDA error to ATTN_ENOMEM / ATTN_ECUDA with a message.
int fail_cuda(cudaError_t e, const char *what);
// The current device index (rejects indices the library does not track).
int current_device(int *dev);
// Device address of the status word on the current device.
int status_ptr(int **out);
// Validates decode arguments and fills `out_args` (sets *empty when B or Hq is 0).
int prep_decode(const attn_tensor *q, const attn_tensor *kcache, const attn_tensor *vcache,
                const attn_tensor *seqlens, const attn_tensor *sinks, int32_t window, float scale,
                int32_t chunk, attn_tensor *out, DecodeArgs *out_args, bool *empty);

}  // namespace attnsink
