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
// (one atomic per block).  A block takes kRowBlock rows of one (batch, head);
// each lane 8 consecutive channels of one row (a row is D/8 lanes, so one warp
// load covers 32/(D/8) rows), every load (LSE included) issued before anything
// else and kept as raw 16-byte words until the sums.  The heads are the fastest
// grid index: blocks that run together read whole [Hq, D] rows of O and dO,
// not one head's slice of many rows.
// The blocks also zero the fp32 dQ, dK and dV accumulators that the main pass
// adds into, while their loads are in flight: rows [R x, R x + R) of batch b
// are one contiguous stretch of each accumulator ([B, L, H, D]), and block
// (x, h, b) zeroes the h-th of Hq equal parts of each stretch, so every block
// stores the same amount.
constexpr int kRowBlock = 64;

template <typename T>
struct Raw8;                                          // 8 channels as loaded
template <>
struct Raw8<__nv_bfloat16> {
  uint4 w;
};
template <>
struct Raw8<float> {
  float4 lo, hi;
};

template <bool kVec, typename T>
__device__ __forceinline__ Raw8<T> load8(const T *p) {
  Raw8<T> r;
  if constexpr (kVec && std::is_same<T, float>::value) {
    r.lo = reinterpret_cast<const float4 *>(p)[0];
    r.hi = reinterpret_cast<const float4 *>(p)[1];
  } else if constexpr (kVec) {
    r.w = *reinterpret_cast<const uint4 *>(p);
  } else if constexpr (std::is_same<T, float>::value) {
    r.lo = make_float4(p[0], p[1], p[2], p[3]);
    r.hi = make_float4(p[4], p[5], p[6], p[7]);
  } else {
    // (bf16 bits gathered two by two: rows with odd strides are only 2-byte aligned)
    const uint16_t *s = reinterpret_cast<const uint16_t *>(p);
    r.w = make_uint4(s[0] | (uint32_t(s[1]) << 16), s[2] | (uint32_t(s[3]) << 16), s[4] | (uint32_t(s[5]) << 16),
                     s[6] | (uint32_t(s[7]) << 16));
  }
  return r;
}

__device__ __forceinline__ void unpack8(const Raw8<__nv_bfloat16> &r, float (&v)[8]) {
  const uint32_t w[4] = {r.w.x, r.w.y, r.w.z, r.w.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    v[2 * e] = __uint_as_float(w[e] << 16);
    v[2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void unpack8(const Raw8<float> &r, float (&v)[8]) {
  v[0] = r.lo.x; v[1] = r.lo.y; v[2] = r.lo.z; v[3] = r.lo.w;
  v[4] = r.hi.x; v[5] = r.hi.y; v[6] = r.hi.z; v[7] = r.hi.w;
}

__device__ __forceinline__ void zero_part(float *base, uint32_t n4, uint32_t part, uint32_t parts) {
  const uint32_t lo = static_cast<uint32_t>(static_cast<uint64_t>(n4) * part / parts);
  const uint32_t hi = static_cast<uint32_t>(static_cast<uint64_t>(n4) * (part + 1) / parts);
  const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
  for (uint32_t e = lo + threadIdx.x; e < hi; e += 256) reinterpret_cast<float4 *>(base)[e] = z;
}

template <typename OT, int D, bool kVec>
__global__ void __launch_bounds__(256) bwd_rows_kernel(const OT *o, const __nv_bfloat16 *dout,
                                                       const float *lse, const float *sinks, float *dsum,
                                                       float *dsink, float *dq_acc, float *dk_acc, float *dv_acc,
                                                       int L, int Hq, int Hkv, int64_t o_sb,
                                                       int64_t o_sl, int64_t o_sh, int64_t d_sb, int64_t d_sl,
                                                       int64_t d_sh, int64_t lse_sb, int64_t lse_sh) {
  constexpr int kLpr = D / 8;                         // lanes per row
  constexpr int kRpl = 32 / kLpr;                     // rows per warp load
  constexpr int kWarpRows = kRowBlock / 8;
  constexpr int kLoads = kWarpRows / kRpl;            // loads per tensor per lane
  const int h = static_cast<int>(blockIdx.x % Hq), x = static_cast<int>(blockIdx.x / Hq), b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nrow = min(kRowBlock, L - x * kRowBlock);
  const int c = (lane % kLpr) * 8;
  const int r0 = x * kRowBlock + warp * kWarpRows + lane / kLpr;   // rows r0 + kRpl k
  Raw8<OT> ov[kLoads];
  Raw8<__nv_bfloat16> dv[kLoads];
#pragma unroll
  for (int k = 0; k < kLoads; ++k) {
    const int i = r0 + kRpl * k;
    if (i < L) {
      ov[k] = load8<kVec>(o + b * o_sb + i * o_sl + h * o_sh + c);
      dv[k] = load8<true>(dout + b * d_sb + i * d_sl + h * d_sh + c);
    }
  }
  const float sink = sinks[h];
  float lv[kLoads];
#pragma unroll
  for (int k = 0; k < kLoads; ++k) {
    const int i = r0 + kRpl * k;
    lv[k] = (lane % kLpr == 0 && i < L && sink != -INFINITY) ? lse[b * lse_sb + h * lse_sh + i] : 0.f;
  }
  {
    const int64_t row0 = static_cast<int64_t>(b) * L + static_cast<int64_t>(x) * kRowBlock;
    zero_part(dq_acc + row0 * Hq * D, static_cast<uint32_t>(nrow * Hq * (D / 4)), h, Hq);
    zero_part(dk_acc + row0 * Hkv * D, static_cast<uint32_t>(nrow * Hkv * (D / 4)), h, Hq);
    zero_part(dv_acc + row0 * Hkv * D, static_cast<uint32_t>(nrow * Hkv * (D / 4)), h, Hq);
  }
  float part = 0.f;
#pragma unroll
  for (int k = 0; k < kLoads; ++k) {
    const int i = r0 + kRpl * k;
    float a = 0.f;
    if (i < L) {
      float x[8], y[8];
      unpack8(ov[k], x);
      unpack8(dv[k], y);
#pragma unroll
      for (int e = 0; e < 8; ++e) a += x[e] * y[e];
    }
#pragma unroll
    for (int off = kLpr / 2; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
    if (lane % kLpr == 0 && i < L) {
      dsum[(static_cast<int64_t>(b) * Hq + h) * L + i] = a;
      if (sink != -INFINITY) part -= __expf(sink - lv[k]) * a;
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
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
// fp32 [B, L, H, D] accumulators -> strided bf16 (dQ; dK and dV after the
// tensor-core main pass): per 8 channels two 16-byte loads and one 16-byte
// store.
// One fp32 accumulator and its strided bf16 destination.
struct ConvertJob {
  const float *acc;
  __nv_bfloat16 *out;
  uint32_t rows, H;
  int64_t s0, s1, s2;
};

// dQ, dK and dV in one launch: the grid strides over the three jobs' 8-channel
// pieces in turn, four pieces per thread per pass (pieces e + u * T, T the
// grid's thread count, so that each warp load stays contiguous), all loads
// issued before the first store.
template <int D>
__global__ void __launch_bounds__(256) bwd_convert_kernel(const ConvertJob j0, const ConvertJob j1,
                                                          const ConvertJob j2, uint32_t L) {
  constexpr uint32_t kPer = D / 8;
  constexpr int kU = 4;
  const uint64_t n0 = static_cast<uint64_t>(j0.rows) * kPer, n1 = static_cast<uint64_t>(j1.rows) * kPer;
  const uint64_t n = n0 + n1 + static_cast<uint64_t>(j2.rows) * kPer;
  const uint64_t T = static_cast<uint64_t>(gridDim.x) * blockDim.x;
  for (uint64_t base = blockIdx.x * static_cast<uint64_t>(blockDim.x) + threadIdx.x; base < n; base += kU * T) {
    float4 x[kU], y[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const uint64_t e = base + u * T;
      if (e < n) {
        // (the job's fields picked one by one, so that none is copied to memory)
        const bool in0 = e < n0, in1 = !in0 && e < n0 + n1;
        const uint64_t el = in0 ? e : (in1 ? e - n0 : e - n0 - n1);
        const float *acc = (in0 ? j0.acc : (in1 ? j1.acc : j2.acc)) + el * 8;
        x[u] = reinterpret_cast<const float4 *>(acc)[0];
        y[u] = reinterpret_cast<const float4 *>(acc)[1];
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const uint64_t e = base + u * T;
      if (e < n) {
        const bool in0 = e < n0, in1 = !in0 && e < n0 + n1;
        const uint64_t el = in0 ? e : (in1 ? e - n0 : e - n0 - n1);
        __nv_bfloat16 *out = in0 ? j0.out : (in1 ? j1.out : j2.out);
        const uint32_t H = in0 ? j0.H : (in1 ? j1.H : j2.H);
        const int64_t s0 = in0 ? j0.s0 : (in1 ? j1.s0 : j2.s0), s1 = in0 ? j0.s1 : (in1 ? j1.s1 : j2.s1),
                      s2 = in0 ? j0.s2 : (in1 ? j1.s2 : j2.s2);
        const uint32_t r = static_cast<uint32_t>(el / kPer), c = static_cast<uint32_t>(el % kPer) * 8;
        const uint32_t h = r % H, bi = r / H;
        const uint32_t i = bi % L, b = bi / L;
        uint4 v;
        v.x = pack_bf16x2(x[u].x, x[u].y);
        v.y = pack_bf16x2(x[u].z, x[u].w);
        v.z = pack_bf16x2(y[u].x, y[u].y);
        v.w = pack_bf16x2(y[u].z, y[u].w);
        *reinterpret_cast<uint4 *>(out + b * s0 + i * s1 + h * s2 + c) = v;
      }
    }
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
  const int64_t row_blocks = static_cast<int64_t>((a.L + kRowBlock - 1) / kRowBlock) * a.Hq;
  if (row_blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
  dim3 rg(static_cast<unsigned>(row_blocks), a.B);
  // a lane's 8 channels are one 16-byte load (two for f32 O) when O's base
  // and strides keep every row's chunks 16-byte aligned; dout's are (its
  // strides are 16-byte multiples)
  const int64_t per16 = a.o_f32 ? 4 : 8;
  const bool ovec = reinterpret_cast<uintptr_t>(a.o) % 16 == 0 && a.o_s[0] % per16 == 0 && a.o_s[1] % per16 == 0 &&
                    a.o_s[2] % per16 == 0;
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
  auto by_dtype = [&](auto dconst) {
    if (a.o_f32) { if (ovec) rows(float{}, dconst, VY{}); else rows(float{}, dconst, VN{}); }
    else { if (ovec) rows(__nv_bfloat16{}, dconst, VY{}); else rows(__nv_bfloat16{}, dconst, VN{}); }
  };
  if (a.D == 128) by_dtype(D128{});
  else by_dtype(D64{});
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = launch_bwd_main_tc(a, dsum, dq_acc, dk_acc, dv_acc, stream)) != cudaSuccess) return e;
  auto job = [&](const float *acc, void *out, int H, const int64_t *s) {
    return ConvertJob{acc, static_cast<__nv_bfloat16 *>(out), static_cast<uint32_t>(static_cast<uint64_t>(a.B) * a.L * H),
                      static_cast<uint32_t>(H), s[0], s[1], s[2]};
  };
  const uint64_t rows64 = static_cast<uint64_t>(a.B) * a.L * (a.Hq + 2 * a.Hkv);
  if (rows64 > 0xFFFFFFFFull) return cudaErrorInvalidValue;
  const uint64_t n = rows64 * (a.D / 8);
  const int blocks = static_cast<int>(n / 256 + 1 < 148 * 4 ? n / 256 + 1 : 148 * 4);   // 4 resident per SM (60 registers)
  const ConvertJob jq = job(dq_acc, a.dq, a.Hq, a.dq_s), jk = job(dk_acc, a.dk, a.Hkv, a.dk_s),
                   jv = job(dv_acc, a.dv, a.Hkv, a.dv_s);
  if (a.D == 128)
    bwd_convert_kernel<128><<<blocks, 256, 0, stream>>>(jq, jk, jv, static_cast<uint32_t>(a.L));
  else
    bwd_convert_kernel<64><<<blocks, 256, 0, stream>>>(jq, jk, jv, static_cast<uint32_t>(a.L));
  return cudaGetLastError();
}

}  // namespace attnsink
