// bwd.cu -- backward pass of sliding-window attention with a learned
// per-head sink: dq, dk, dv and dsink for the loss sum(dout * O).
//
// Gradient of the sink (page "Dao-AILab/flash-attention" contributor guide,
// issue #2969: the sink's gradient is to be formed from the unrounded O).
// With P_ij = exp(s_ij - LSE_i), P_sink,i = exp(sink - LSE_i) and
// Dsum_i = dO_i . O_i:
//   dV_j    = sum_i P_ij dO_i
//   dP_ij   = dO_i . v_j
//   dS_ij   = P_ij (dP_ij - Dsum_i)
//   dQ_i    = scale * sum_j dS_ij k_j
//   dK_j    = scale * sum_i dS_ij q_i
//   dsink_h = -sum_i P_sink,i Dsum_i
// (the sink takes mass from every content probability in proportion, so its
// gradient is minus its probability times the row's dO . O).
//
// Launches: a row kernel forms Dsum (from O as given: bf16 or, for the exact
// form, f32) and the sink gradient; the tensor-core main pass (bwd_tc.cu)
// sums dQ, dK and dV in fp32 workspaces; one conversion kernel writes them
// as bf16.
#include <math.h>

#include <type_traits>

#include "kernels.h"
#include "ptx.cuh"

namespace attnsink {
namespace {


// ------------------------------------------------------------------ rows
// Dsum[b, h, i] = dO . O for every row, and dsink[h] -= exp(sink - LSE) * Dsum
// (one atomic per block).  The block also zeroes its rows of the fp32 dQ
// accumulator, and (blocks of the first Hkv heads) those of dK and dV, which
// the main pass then adds into.  A block takes 64 rows of one (batch, head); each
// warp takes 8 of them with every load issued before the first sum, each lane
// D/32 consecutive channels (vector loads when the rows are aligned).
template <int E, bool kVec, typename T>
__device__ __forceinline__ void load_row(const T *p, float (&v)[E]) {
  if constexpr (kVec && std::is_same<T, float>::value && E == 4) {
    const float4 x = *reinterpret_cast<const float4 *>(p);
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
  } else if constexpr (kVec && std::is_same<T, float>::value && E == 2) {
    const float2 x = *reinterpret_cast<const float2 *>(p);
    v[0] = x.x; v[1] = x.y;
  } else if constexpr (kVec && !std::is_same<T, float>::value && E == 4) {
    const uint2 x = *reinterpret_cast<const uint2 *>(p);
    v[0] = __uint_as_float(x.x << 16); v[1] = __uint_as_float(x.x & 0xFFFF0000u);
    v[2] = __uint_as_float(x.y << 16); v[3] = __uint_as_float(x.y & 0xFFFF0000u);
  } else if constexpr (kVec && !std::is_same<T, float>::value && E == 2) {
    const uint32_t x = *reinterpret_cast<const uint32_t *>(p);
    v[0] = __uint_as_float(x << 16); v[1] = __uint_as_float(x & 0xFFFF0000u);
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) v[e] = static_cast<float>(p[e]);
  }
}

template <typename OT, int D, bool kVec>
__global__ void __launch_bounds__(256) bwd_rows_kernel(const OT *o, const __nv_bfloat16 *dout,
                                                       const float *lse, const float *sinks, float *dsum,
                                                       float *dsink, float *dq_acc, float *dk_acc, float *dv_acc,
                                                       int L, int Hq, int Hkv, int64_t o_sb,
                                                       int64_t o_sl, int64_t o_sh, int64_t d_sb, int64_t d_sl,
                                                       int64_t d_sh, int64_t lse_sb, int64_t lse_sh) {
  constexpr int E = D / 32;
  const int h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i0 = blockIdx.x * 64 + warp;             // rows i0, i0 + 8, ..., i0 + 56
  {
    // zero this block's accumulator rows (16-byte stores, a row's D floats
    // by consecutive threads)
    const int nrow = min(64, L - static_cast<int>(blockIdx.x) * 64);
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    const int64_t row0 = static_cast<int64_t>(b) * L + static_cast<int64_t>(blockIdx.x) * 64;
    for (int e = threadIdx.x; e < nrow * (D / 4); e += 256) {
      const int r = e / (D / 4), c = (e - r * (D / 4)) * 4;
      *reinterpret_cast<float4 *>(dq_acc + ((row0 + r) * Hq + h) * D + c) = z;
      if (h < Hkv) {
        *reinterpret_cast<float4 *>(dk_acc + ((row0 + r) * Hkv + h) * D + c) = z;
        *reinterpret_cast<float4 *>(dv_acc + ((row0 + r) * Hkv + h) * D + c) = z;
      }
    }
  }
  float acc[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int i = i0 + 8 * k;
    float a = 0.f;
    if (i < L) {
      float ov[E], dv[E];
      load_row<E, kVec>(o + b * o_sb + i * o_sl + h * o_sh + lane * E, ov);
      load_row<E, kVec>(dout + b * d_sb + i * d_sl + h * d_sh + lane * E, dv);
#pragma unroll
      for (int e = 0; e < E; ++e) a += ov[e] * dv[e];
    }
    acc[k] = a;
  }
#pragma unroll
  for (int k = 0; k < 8; ++k)
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc[k] += __shfl_xor_sync(0xffffffffu, acc[k], off);
  // lane k < 8 finishes row i0 + 8k
  float mine = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) mine = (lane == k) ? acc[k] : mine;
  const int i = i0 + 8 * lane;
  const float sink = sinks[h];
  float part = 0.f;
  if (lane < 8 && i < L) {
    dsum[(static_cast<int64_t>(b) * Hq + h) * L + i] = mine;
    if (sink != -INFINITY) part = -__expf(sink - lse[b * lse_sb + h * lse_sh + i]) * mine;
  }
#pragma unroll
  for (int off = 4; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
  __shared__ float red[8];
  if (lane == 0) red[warp] = part;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < 8; ++w) t += red[w];
    if (t != 0.f) atomicAdd(&dsink[h], t);
  }
}

// ------------------------------------------------------------------ dQ out
// fp32 [B, L, H, D] accumulator -> strided bf16 (dQ; dK and dV after the
// tensor-core main pass): one thread per 8 channels, two 16-byte loads and
// one 16-byte store.
// One fp32 accumulator and its strided bf16 destination.
struct ConvertJob {
  const float *acc;
  __nv_bfloat16 *out;
  uint32_t rows, H;
  int64_t s0, s1, s2;
};

// dQ, dK and dV in one launch: the grid strides over the three jobs' 8-channel
// pieces in turn.
template <int D>
__global__ void bwd_convert_kernel(const ConvertJob j0, const ConvertJob j1, const ConvertJob j2, uint32_t L) {
  constexpr uint32_t kPer = D / 8;
  const uint64_t n0 = static_cast<uint64_t>(j0.rows) * kPer, n1 = static_cast<uint64_t>(j1.rows) * kPer;
  const uint64_t n = n0 + n1 + static_cast<uint64_t>(j2.rows) * kPer;
  for (uint64_t e = blockIdx.x * static_cast<uint64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
    // (the job's fields picked one by one, so that none is copied to memory)
    const bool in0 = e < n0, in1 = !in0 && e < n0 + n1;
    const uint64_t el = in0 ? e : (in1 ? e - n0 : e - n0 - n1);
    const float *acc = in0 ? j0.acc : (in1 ? j1.acc : j2.acc);
    __nv_bfloat16 *out = in0 ? j0.out : (in1 ? j1.out : j2.out);
    const uint32_t H = in0 ? j0.H : (in1 ? j1.H : j2.H);
    const int64_t s0 = in0 ? j0.s0 : (in1 ? j1.s0 : j2.s0), s1 = in0 ? j0.s1 : (in1 ? j1.s1 : j2.s1),
                  s2 = in0 ? j0.s2 : (in1 ? j1.s2 : j2.s2);
    const uint32_t r = static_cast<uint32_t>(el / kPer), c = static_cast<uint32_t>(el % kPer) * 8;
    const uint32_t h = r % H, bi = r / H;
    const uint32_t i = bi % L, b = bi / L;
    const float4 x = *reinterpret_cast<const float4 *>(acc + static_cast<uint64_t>(r) * D + c);
    const float4 y = *reinterpret_cast<const float4 *>(acc + static_cast<uint64_t>(r) * D + c + 4);
    uint4 v;
    v.x = pack_bf16x2(x.x, x.y);
    v.y = pack_bf16x2(x.z, x.w);
    v.z = pack_bf16x2(y.x, y.y);
    v.w = pack_bf16x2(y.z, y.w);
    *reinterpret_cast<uint4 *>(out + b * s0 + i * s1 + h * s2 + c) = v;
  }
}

}  // namespace

// Workspace: the fp32 dQ accumulator [B, L, Hq, D], Dsum [B, Hq, L], and
// fp32 dK, dV accumulators [B, L, Hkv, D].
namespace {
size_t align256(size_t n) { return (n + 255) / 256 * 256; }
}  // namespace

size_t bwd_workspace_bytes(const BwdArgs &a) {
  const size_t acc = sizeof(float) * static_cast<size_t>(a.B) * a.L * a.Hq * a.D;
  const size_t ds = sizeof(float) * static_cast<size_t>(a.B) * a.Hq * a.L;
  const size_t kv = 2 * align256(sizeof(float) * static_cast<size_t>(a.B) * a.L * a.Hkv * a.D);
  return align256(acc) + align256(ds) + kv;
}

cudaError_t launch_bwd(const BwdArgs &a, void *workspace, cudaStream_t stream) {
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  float *dq_acc = reinterpret_cast<float *>(ws);
  const size_t acc_bytes = sizeof(float) * static_cast<size_t>(a.B) * a.L * a.Hq * a.D;
  float *dsum = reinterpret_cast<float *>(ws + align256(acc_bytes));
  const size_t ds_bytes = sizeof(float) * static_cast<size_t>(a.B) * a.Hq * a.L;
  const size_t kv_bytes = sizeof(float) * static_cast<size_t>(a.B) * a.L * a.Hkv * a.D;
  float *dk_acc = reinterpret_cast<float *>(ws + align256(acc_bytes) + align256(ds_bytes));
  float *dv_acc = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(dk_acc) + align256(kv_bytes));
  // (the row kernel zeroes the dQ, dK and dV accumulators)
  cudaError_t e = cudaMemsetAsync(a.dsink, 0, sizeof(float) * a.Hq, stream);
  if (e != cudaSuccess) return e;
  dim3 rg((a.L + 63) / 64, a.Hq, a.B);
  // vector loads of O need its rows aligned to the per-lane chunk (bf16 rows
  // are: their strides and base are 16-byte multiples)
  const int E = a.D / 32;
  const int eb = a.o_f32 ? 4 : 2;
  const bool ovec = reinterpret_cast<uintptr_t>(a.o) % (E * eb) == 0 && a.o_s[0] % E == 0 && a.o_s[1] % E == 0 &&
                    a.o_s[2] % E == 0;
  auto rows = [&](auto ot, auto dconst, auto vec) {
    using OT = decltype(ot);
    bwd_rows_kernel<OT, decltype(dconst)::value, decltype(vec)::value><<<rg, 256, 0, stream>>>(
        static_cast<const OT *>(a.o), static_cast<const __nv_bfloat16 *>(a.dout), a.lse, a.sinks, dsum, a.dsink,
        dq_acc, dk_acc, dv_acc, a.L, a.Hq, a.Hkv, a.o_s[0], a.o_s[1], a.o_s[2], a.do_s[0], a.do_s[1], a.do_s[2], a.lse_s[0], a.lse_s[1]);
  };
  using D64 = std::integral_constant<int, 64>;
  using D128 = std::integral_constant<int, 128>;
  using VY = std::true_type;
  using VN = std::false_type;
  if (a.D == 128) {
    if (a.o_f32) { if (ovec) rows(float{}, D128{}, VY{}); else rows(float{}, D128{}, VN{}); }
    else rows(__nv_bfloat16{}, D128{}, VY{});
  } else {
    if (a.o_f32) { if (ovec) rows(float{}, D64{}, VY{}); else rows(float{}, D64{}, VN{}); }
    else rows(__nv_bfloat16{}, D64{}, VY{});
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = launch_bwd_main_tc(a, dsum, dq_acc, dk_acc, dv_acc, stream)) != cudaSuccess) return e;
  auto job = [&](const float *acc, void *out, int H, const int64_t *s) {
    return ConvertJob{acc, static_cast<__nv_bfloat16 *>(out), static_cast<uint32_t>(static_cast<uint64_t>(a.B) * a.L * H),
                      static_cast<uint32_t>(H), s[0], s[1], s[2]};
  };
  const uint64_t rows64 = static_cast<uint64_t>(a.B) * a.L * (a.Hq + 2 * a.Hkv);
  if (rows64 > 0xFFFFFFFFull) return cudaErrorInvalidValue;
  const uint64_t n = rows64 * (a.D / 8);
  const int blocks = static_cast<int>(n / 256 + 1 < 148 * 8 ? n / 256 + 1 : 148 * 8);
  const ConvertJob jq = job(dq_acc, a.dq, a.Hq, a.dq_s), jk = job(dk_acc, a.dk, a.Hkv, a.dk_s),
                   jv = job(dv_acc, a.dv, a.Hkv, a.dv_s);
  if (a.D == 128)
    bwd_convert_kernel<128><<<blocks, 256, 0, stream>>>(jq, jk, jv, static_cast<uint32_t>(a.L));
  else
    bwd_convert_kernel<64><<<blocks, 256, 0, stream>>>(jq, jk, jv, static_cast<uint32_t>(a.L));
  return cudaGetLastError();
}

}  // namespace attnsink
