// fwd_cudacore.cu -- the prefill forward on plain CUDA cores in fp32, one warp
// per output row.  It shares the definition (page "cf-1.com/news/6055759":
// sliding-window softmax with one learned sink logit per head, the running
// maximum rebased on the sink at the end as in its fix 2) but nothing else
// with the tensor-core kernel, so the two can be checked against each other
// on sizes where the fp64 oracle would be too slow.  Not a fast path.
#include <math.h>

#include <cuda_bf16.h>

#include "kernels.h"

namespace attnsink {
namespace {

struct RefParams {
  const __nv_bfloat16 *q, *k, *v;
  const float *sinks;
  __nv_bfloat16 *out;
  float *lse;
  int B, L, Hq, Hkv, W;
  float scale_log2;
  int64_t q_s[3], k_s[3], v_s[3], o_s[3], lse_s[2];
};

template <int DPL>  // channels per lane: D = 32 * DPL
__global__ void __launch_bounds__(256) fwd_cudacore_kernel(const RefParams p) {
  const int64_t warp_global = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t rows = static_cast<int64_t>(p.B) * p.L * p.Hq;
  if (warp_global >= rows) return;
  const int h = static_cast<int>(warp_global % p.Hq);
  const int i = static_cast<int>((warp_global / p.Hq) % p.L);
  const int b = static_cast<int>(warp_global / (static_cast<int64_t>(p.Hq) * p.L));
  const int hk = h / (p.Hq / p.Hkv);

  const __nv_bfloat16 *qr = p.q + b * p.q_s[0] + i * p.q_s[1] + h * p.q_s[2];
  float qv[DPL], acc[DPL];
#pragma unroll
  for (int t = 0; t < DPL; ++t) {
    qv[t] = __bfloat162float(qr[lane + 32 * t]);
    acc[t] = 0.f;
  }
  float m = -INFINITY, l = 0.f;  // log2-domain running max and denominator
  const int lo = max(0, i - p.W + 1);
  for (int j = lo; j <= i; ++j) {
    const __nv_bfloat16 *kr = p.k + b * p.k_s[0] + static_cast<int64_t>(j) * p.k_s[1] + hk * p.k_s[2];
    const __nv_bfloat16 *vr = p.v + b * p.v_s[0] + static_cast<int64_t>(j) * p.v_s[1] + hk * p.v_s[2];
    float dot = 0.f;
#pragma unroll
    for (int t = 0; t < DPL; ++t) dot = fmaf(qv[t], __bfloat162float(kr[lane + 32 * t]), dot);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
    const float x = dot * p.scale_log2;
    if (x > m) {
      const float a = exp2f(m - x);
      l *= a;
#pragma unroll
      for (int t = 0; t < DPL; ++t) acc[t] *= a;
      m = x;
    }
    const float pj = exp2f(x - m);
    l += pj;
#pragma unroll
    for (int t = 0; t < DPL; ++t) acc[t] = fmaf(pj, __bfloat162float(vr[lane + 32 * t]), acc[t]);
  }
  const float sink2 = p.sinks[h] * 1.4426950408889634f;
  const float nm = fmaxf(m, sink2);
  const float r = (m == -INFINITY) ? 0.f : exp2f(m - nm);
  const float l2 = l * r + ((sink2 == -INFINITY) ? 0.f : exp2f(sink2 - nm));
  const float sc = (l2 > 0.f) ? r / l2 : 0.f;
  __nv_bfloat16 *orow = p.out + b * p.o_s[0] + i * p.o_s[1] + h * p.o_s[2];
#pragma unroll
  for (int t = 0; t < DPL; ++t) orow[lane + 32 * t] = __float2bfloat16_rn(acc[t] * sc);
  if (p.lse != nullptr && lane == 0)
    p.lse[b * p.lse_s[0] + h * p.lse_s[1] + i] = (l2 > 0.f) ? (nm + log2f(l2)) * 0.6931471805599453f
                                                             : -INFINITY;
}

template <int DPL>
cudaError_t launch(const RefParams &p, cudaStream_t stream) {
  const int64_t rows = static_cast<int64_t>(p.B) * p.L * p.Hq;
  const int64_t blocks = (rows * 32 + 255) / 256;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  fwd_cudacore_kernel<DPL><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_cudacore(const FwdArgs &a, cudaStream_t stream) {
  RefParams p;
  p.q = static_cast<const __nv_bfloat16 *>(a.q);
  p.k = static_cast<const __nv_bfloat16 *>(a.k);
  p.v = static_cast<const __nv_bfloat16 *>(a.v);
  p.sinks = a.sinks;
  p.out = static_cast<__nv_bfloat16 *>(a.out);
  p.lse = a.lse;
  p.B = a.B;
  p.L = a.L;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.W = a.W;
  p.scale_log2 = static_cast<float>(static_cast<double>(a.scale) * 1.4426950408889634);
  for (int t = 0; t < 3; ++t) {
    p.q_s[t] = a.q_s[t];
    p.k_s[t] = a.k_s[t];
    p.v_s[t] = a.v_s[t];
    p.o_s[t] = a.o_s[t];
  }
  p.lse_s[0] = a.lse_s[0];
  p.lse_s[1] = a.lse_s[1];
  switch (a.D) {
    case 32: return launch<1>(p, stream);
    case 64: return launch<2>(p, stream);
    case 96: return launch<3>(p, stream);
    case 128: return launch<4>(p, stream);
    case 160: return launch<5>(p, stream);
    case 192: return launch<6>(p, stream);
    case 224: return launch<7>(p, stream);
    case 256: return launch<8>(p, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace attnsink
