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
// Three launches: a row kernel forms Dsum (from O as given: bf16 or, for the
// exact form, f32) and the sink gradient; the main kernel takes one block of
// 64 keys of one kv head and walks every query block of every query head of
// the group that sees those keys, with five warp-level bf16 tensor-core
// products per step (S^T = K Q^T, dV += P^T dO, dP^T = V dO^T, dK += dS^T Q,
// dQ += dS K); dK and dV stay in registers, dQ is summed in fp32 in a
// workspace by atomic adds and converted to bf16 by the third launch.
#include <math.h>

#include <type_traits>

#include "kernels.h"
#include "ptx.cuh"

namespace attnsink {
namespace {

constexpr int kBK = 64;          // keys per block (16 per warp)
constexpr int kBQ = 64;          // query rows per step
constexpr int kWarps = 4;
constexpr float kLog2e = 1.4426950408889634f;

// Swizzled 16-bit tile of R rows: 64-column chunks of R x 128 bytes; row r's
// 16-byte unit u sits at unit u ^ (r & 7).  Byte offset of (row, col).
template <int R>
__device__ __forceinline__ uint32_t toff(int row, int col) {
  return static_cast<uint32_t>((col >> 6) * (R * 128) + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) +
                               (col & 7) * 2);
}

// Copies rows [r0, r0 + R) of one head of a [.., L, H, D] bf16 tensor into a
// swizzled tile (rows at or past L become zeros).
template <int R, int D>
__device__ __forceinline__ void load_tile(uint8_t *tile, const __nv_bfloat16 *base, int64_t row_stride,
                                          int r0, int L) {
  constexpr int kUnits = R * D / 8;   // 16-byte units
  for (int e = threadIdx.x; e < kUnits; e += kWarps * 32) {
    const int row = e / (D / 8), u = e % (D / 8);
    uint4 x = make_uint4(0, 0, 0, 0);
    if (r0 + row < L) x = *reinterpret_cast<const uint4 *>(base + static_cast<int64_t>(r0 + row) * row_stride + u * 8);
    *reinterpret_cast<uint4 *>(tile + toff<R>(row, u * 8)) = x;
  }
}

struct BwdParams {
  const __nv_bfloat16 *q, *k, *v, *dout;
  const float *lse, *dsum;
  float *dq_acc;
  __nv_bfloat16 *dk, *dv;
  int B, L, Hq, Hkv, W;
  float scale, scale_log2;
  int64_t q_s[3], k_s[3], v_s[3], do_s[3], dk_s[3], dv_s[3], lse_s[2];
};

// ------------------------------------------------------------------ rows
// Dsum[b, h, i] = dO . O for every row, and dsink[h] -= exp(sink - LSE) * Dsum
// (one atomic per block).  A block takes 64 rows of one (batch, head); each
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
                                                       float *dsink, int L, int Hq, int64_t o_sb,
                                                       int64_t o_sl, int64_t o_sh, int64_t d_sb, int64_t d_sl,
                                                       int64_t d_sh, int64_t lse_sb, int64_t lse_sh) {
  constexpr int E = D / 32;
  const int h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i0 = blockIdx.x * 64 + warp;             // rows i0, i0 + 8, ..., i0 + 56
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

// ------------------------------------------------------------------ main
template <int D>
__global__ void __launch_bounds__(kWarps * 32) bwd_main_kernel(const BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  constexpr int kTile = kBK * D * 2;
  uint8_t *sK = smem, *sV = sK + kTile, *sQ = sV + kTile, *sO = sQ + kTile;   // sO: dO tile
  uint8_t *sS = sO + kTile;                                                    // dS^T [keys x queries]
  float *sLse = reinterpret_cast<float *>(sS + kBK * kBQ * 2);                 // log2 units
  float *sDs = sLse + kBQ;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g8 = lane >> 2, tig = lane & 3;
  const int j0 = blockIdx.x * kBK, hk = blockIdx.y, b = blockIdx.z;
  const int G = p.Hq / p.Hkv;
  const int key_w = warp * 16;               // this warp's keys within the block

  load_tile<kBK, D>(sK, p.k + b * p.k_s[0] + hk * p.k_s[2], p.k_s[1], j0, p.L);
  load_tile<kBK, D>(sV, p.v + b * p.v_s[0] + hk * p.v_s[2], p.v_s[1], j0, p.L);

  float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
  for (int n = 0; n < D / 8; ++n)
#pragma unroll
    for (int f = 0; f < 4; ++f) dk[n][f] = dv[n][f] = 0.f;

  // queries that see a key of [j0, j0 + 63]: rows [j0, j0 + 63 + W - 1]
  const int q_lo = j0 / kBQ;
  const int q_hi = min(p.L - 1, j0 + kBK - 1 + min(p.W - 1, p.L)) / kBQ;
  for (int hh = 0; hh < G; ++hh) {
    const int h = hk * G + hh;
    for (int qb = q_lo; qb <= q_hi; ++qb) {
      const int i0 = qb * kBQ;
      __syncthreads();                       // previous step's tiles fully read
      load_tile<kBQ, D>(sQ, p.q + b * p.q_s[0] + h * p.q_s[2], p.q_s[1], i0, p.L);
      load_tile<kBQ, D>(sO, p.dout + b * p.do_s[0] + h * p.do_s[2], p.do_s[1], i0, p.L);
      for (int t = threadIdx.x; t < kBQ; t += kWarps * 32) {
        const int i = i0 + t;
        sLse[t] = i < p.L ? p.lse[b * p.lse_s[0] + h * p.lse_s[1] + i] * kLog2e : INFINITY;
        sDs[t] = i < p.L ? p.dsum[(static_cast<int64_t>(b) * p.Hq + h) * p.L + i] : 0.f;
      }
      __syncthreads();

      // ---- S^T[16 keys x 64 queries] = K_w Q^T ----
      float st[kBQ / 8][4];
#pragma unroll
      for (int n = 0; n < kBQ / 8; ++n)
#pragma unroll
        for (int f = 0; f < 4; ++f) st[n][f] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(smem_u32(sK) + toff<kBK>(key_w + (lane & 7) + ((lane >> 3) & 1) * 8, kk * 16 + (lane >> 4) * 8),
                    a0, a1, a2, a3);
#pragma unroll
        for (int n = 0; n < kBQ / 8; n += 2) {
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4(smem_u32(sQ) + toff<kBQ>((n + (lane >> 4)) * 8 + (lane & 7), kk * 16 + ((lane >> 3) & 1) * 8),
                      b0, b1, b2, b3);
          mma_bf16_16816(st[n], a0, a1, a2, a3, b0, b1);
          mma_bf16_16816(st[n + 1], a0, a1, a2, a3, b2, b3);
        }
      }
      // ---- P^T = exp(s - LSE) on the visible (key, query) pairs ----
      const int jr0 = j0 + key_w + g8, jr1 = jr0 + 8;   // this thread's key rows
#pragma unroll
      for (int n = 0; n < kBQ / 8; ++n) {
#pragma unroll
        for (int f = 0; f < 4; ++f) {
          const int c = n * 8 + 2 * tig + (f & 1);
          const int i = i0 + c, j = (f < 2) ? jr0 : jr1;
          const bool vis = i < p.L && j <= i && j >= i - p.W + 1;
          st[n][f] = vis ? ex2_approx(st[n][f] * p.scale_log2 - sLse[c]) : 0.f;
        }
      }
      // ---- dV_w += P^T dO ----
#pragma unroll
      for (int ks = 0; ks < kBQ / 16; ++ks) {
        const uint32_t a0 = pack_bf16x2(st[2 * ks][0], st[2 * ks][1]);
        const uint32_t a1 = pack_bf16x2(st[2 * ks][2], st[2 * ks][3]);
        const uint32_t a2 = pack_bf16x2(st[2 * ks + 1][0], st[2 * ks + 1][1]);
        const uint32_t a3 = pack_bf16x2(st[2 * ks + 1][2], st[2 * ks + 1][3]);
#pragma unroll
        for (int n = 0; n < D / 8; n += 2) {
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4_trans(smem_u32(sO) + toff<kBQ>(ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8, n * 8 + (lane >> 4) * 8),
                            b0, b1, b2, b3);
          mma_bf16_16816(dv[n], a0, a1, a2, a3, b0, b1);
          mma_bf16_16816(dv[n + 1], a0, a1, a2, a3, b2, b3);
        }
      }
      // ---- dP^T[16 keys x 64 queries] = V_w dO^T; dS^T = P^T (dP^T - Dsum) ----
      float dp[kBQ / 8][4];
#pragma unroll
      for (int n = 0; n < kBQ / 8; ++n)
#pragma unroll
        for (int f = 0; f < 4; ++f) dp[n][f] = 0.f;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(smem_u32(sV) + toff<kBK>(key_w + (lane & 7) + ((lane >> 3) & 1) * 8, kk * 16 + (lane >> 4) * 8),
                    a0, a1, a2, a3);
#pragma unroll
        for (int n = 0; n < kBQ / 8; n += 2) {
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4(smem_u32(sO) + toff<kBQ>((n + (lane >> 4)) * 8 + (lane & 7), kk * 16 + ((lane >> 3) & 1) * 8),
                      b0, b1, b2, b3);
          mma_bf16_16816(dp[n], a0, a1, a2, a3, b0, b1);
          mma_bf16_16816(dp[n + 1], a0, a1, a2, a3, b2, b3);
        }
      }
#pragma unroll
      for (int n = 0; n < kBQ / 8; ++n)
#pragma unroll
        for (int f = 0; f < 4; ++f) st[n][f] *= dp[n][f] - sDs[n * 8 + 2 * tig + (f & 1)];   // now dS^T
      // ---- dK_w += dS^T Q; dS^T (bf16) to shared memory for dQ ----
#pragma unroll
      for (int ks = 0; ks < kBQ / 16; ++ks) {
        const uint32_t a0 = pack_bf16x2(st[2 * ks][0], st[2 * ks][1]);
        const uint32_t a1 = pack_bf16x2(st[2 * ks][2], st[2 * ks][3]);
        const uint32_t a2 = pack_bf16x2(st[2 * ks + 1][0], st[2 * ks + 1][1]);
        const uint32_t a3 = pack_bf16x2(st[2 * ks + 1][2], st[2 * ks + 1][3]);
        *reinterpret_cast<uint32_t *>(sS + toff<kBK>(key_w + g8, ks * 16 + 2 * tig)) = a0;
        *reinterpret_cast<uint32_t *>(sS + toff<kBK>(key_w + g8 + 8, ks * 16 + 2 * tig)) = a1;
        *reinterpret_cast<uint32_t *>(sS + toff<kBK>(key_w + g8, ks * 16 + 8 + 2 * tig)) = a2;
        *reinterpret_cast<uint32_t *>(sS + toff<kBK>(key_w + g8 + 8, ks * 16 + 8 + 2 * tig)) = a3;
#pragma unroll
        for (int n = 0; n < D / 8; n += 2) {
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4_trans(smem_u32(sQ) + toff<kBQ>(ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8, n * 8 + (lane >> 4) * 8),
                            b0, b1, b2, b3);
          mma_bf16_16816(dk[n], a0, a1, a2, a3, b0, b1);
          mma_bf16_16816(dk[n + 1], a0, a1, a2, a3, b2, b3);
        }
      }
      __syncthreads();                       // dS^T of all four warps in shared memory
      // ---- dQ[16 queries of this warp x D] = dS K, summed into the fp32 workspace ----
      {
        const int qw = warp * 16;            // this warp's query rows within the step
        float dq[D / 8][4];
#pragma unroll
        for (int n = 0; n < D / 8; ++n)
#pragma unroll
          for (int f = 0; f < 4; ++f) dq[n][f] = 0.f;
#pragma unroll
        for (int ks = 0; ks < kBK / 16; ++ks) {
          // A = dS (query rows, key columns) from the dS^T tile, transposed
          const int m = lane >> 3;
          uint32_t a0, a1, a2, a3;
          ldmatrix_x4_trans(smem_u32(sS) + toff<kBK>(ks * 16 + (lane & 7) + (m >= 2 ? 8 : 0), qw + ((m & 1) ? 8 : 0)),
                            a0, a1, a2, a3);
#pragma unroll
          for (int n = 0; n < D / 8; n += 2) {
            uint32_t b0, b1, b2, b3;
            ldmatrix_x4_trans(smem_u32(sK) + toff<kBK>(ks * 16 + (lane & 7) + ((lane >> 3) & 1) * 8, n * 8 + (lane >> 4) * 8),
                              b0, b1, b2, b3);
            mma_bf16_16816(dq[n], a0, a1, a2, a3, b0, b1);
            mma_bf16_16816(dq[n + 1], a0, a1, a2, a3, b2, b3);
          }
        }
        const int ia = i0 + qw + g8, ib = ia + 8;
        float *base = p.dq_acc + ((static_cast<int64_t>(b) * p.L) * p.Hq + h) * D;
#pragma unroll
        for (int n = 0; n < D / 8; ++n) {
          const int d = n * 8 + 2 * tig;
          if (ia < p.L) {
            atomicAdd(base + (static_cast<int64_t>(ia) * p.Hq) * D + d, dq[n][0] * p.scale);
            atomicAdd(base + (static_cast<int64_t>(ia) * p.Hq) * D + d + 1, dq[n][1] * p.scale);
          }
          if (ib < p.L) {
            atomicAdd(base + (static_cast<int64_t>(ib) * p.Hq) * D + d, dq[n][2] * p.scale);
            atomicAdd(base + (static_cast<int64_t>(ib) * p.Hq) * D + d + 1, dq[n][3] * p.scale);
          }
        }
      }
    }
  }
  // ---- dK (times scale) and dV of this warp's 16 keys ----
  const int ja = j0 + key_w + g8, jb = ja + 8;
#pragma unroll
  for (int n = 0; n < D / 8; ++n) {
    const int d = n * 8 + 2 * tig;
    if (ja < p.L) {
      *reinterpret_cast<uint32_t *>(p.dk + b * p.dk_s[0] + static_cast<int64_t>(ja) * p.dk_s[1] + hk * p.dk_s[2] + d) =
          pack_bf16x2(dk[n][0] * p.scale, dk[n][1] * p.scale);
      *reinterpret_cast<uint32_t *>(p.dv + b * p.dv_s[0] + static_cast<int64_t>(ja) * p.dv_s[1] + hk * p.dv_s[2] + d) =
          pack_bf16x2(dv[n][0], dv[n][1]);
    }
    if (jb < p.L) {
      *reinterpret_cast<uint32_t *>(p.dk + b * p.dk_s[0] + static_cast<int64_t>(jb) * p.dk_s[1] + hk * p.dk_s[2] + d) =
          pack_bf16x2(dk[n][2] * p.scale, dk[n][3] * p.scale);
      *reinterpret_cast<uint32_t *>(p.dv + b * p.dv_s[0] + static_cast<int64_t>(jb) * p.dv_s[1] + hk * p.dv_s[2] + d) =
          pack_bf16x2(dv[n][2], dv[n][3]);
    }
  }
}

// ------------------------------------------------------------------ dQ out
// fp32 [B, L, H, D] accumulator -> strided bf16 (dQ; dK and dV after the
// tensor-core main pass): one thread per 8 channels, two 16-byte loads and
// one 16-byte store.
template <int D>
__global__ void bwd_convert_kernel(const float *acc, __nv_bfloat16 *out, uint32_t rows, uint32_t H, uint32_t L,
                                   int64_t s0, int64_t s1, int64_t s2) {
  constexpr uint32_t kPer = D / 8;
  const uint64_t n = static_cast<uint64_t>(rows) * kPer;
  for (uint64_t e = blockIdx.x * static_cast<uint64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
    const uint32_t r = static_cast<uint32_t>(e / kPer), c = static_cast<uint32_t>(e % kPer) * 8;
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

template <int D>
cudaError_t launch_main(const BwdArgs &a, float *dq_acc, const float *dsum, cudaStream_t stream) {
  BwdParams p;
  p.q = static_cast<const __nv_bfloat16 *>(a.q);
  p.k = static_cast<const __nv_bfloat16 *>(a.k);
  p.v = static_cast<const __nv_bfloat16 *>(a.v);
  p.dout = static_cast<const __nv_bfloat16 *>(a.dout);
  p.lse = a.lse;
  p.dsum = dsum;
  p.dq_acc = dq_acc;
  p.dk = static_cast<__nv_bfloat16 *>(a.dk);
  p.dv = static_cast<__nv_bfloat16 *>(a.dv);
  p.B = a.B;
  p.L = a.L;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.W = a.W;
  p.scale = a.scale;
  p.scale_log2 = static_cast<float>(static_cast<double>(a.scale) * 1.4426950408889634);
  for (int d = 0; d < 3; ++d) {
    p.q_s[d] = a.q_s[d];
    p.k_s[d] = a.k_s[d];
    p.v_s[d] = a.v_s[d];
    p.do_s[d] = a.do_s[d];
    p.dk_s[d] = a.dk_s[d];
    p.dv_s[d] = a.dv_s[d];
  }
  p.lse_s[0] = a.lse_s[0];
  p.lse_s[1] = a.lse_s[1];
  const int smem = 4 * kBK * D * 2 + kBK * kBQ * 2 + 2 * kBQ * 4 + 1024;
  auto kern = bwd_main_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.L + kBK - 1) / kBK, a.Hkv, a.B);
  kern<<<grid, kWarps * 32, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

// Workspace: the fp32 dQ accumulator [B, L, Hq, D], Dsum [B, Hq, L], and for
// D = 128 (the tensor-core main pass) fp32 dK, dV accumulators [B, L, Hkv, D].
namespace {
size_t align256(size_t n) { return (n + 255) / 256 * 256; }
}  // namespace

size_t bwd_workspace_bytes(const BwdArgs &a) {
  const size_t acc = sizeof(float) * static_cast<size_t>(a.B) * a.L * a.Hq * a.D;
  const size_t ds = sizeof(float) * static_cast<size_t>(a.B) * a.Hq * a.L;
  const size_t kv = a.D == 128 ? 2 * align256(sizeof(float) * static_cast<size_t>(a.B) * a.L * a.Hkv * a.D) : 0;
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
  const bool tc = a.D == 128;
  cudaError_t e = cudaMemsetAsync(dq_acc, 0, acc_bytes, stream);
  if (e != cudaSuccess) return e;
  if (tc && (e = cudaMemsetAsync(dk_acc, 0, align256(kv_bytes) + kv_bytes, stream)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(a.dsink, 0, sizeof(float) * a.Hq, stream)) != cudaSuccess) return e;
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
        a.L, a.Hq, a.o_s[0], a.o_s[1], a.o_s[2], a.do_s[0], a.do_s[1], a.do_s[2], a.lse_s[0], a.lse_s[1]);
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
  switch (a.D) {
    case 64: e = launch_main<64>(a, dq_acc, dsum, stream); break;
    case 128: e = launch_bwd_main_tc(a, dsum, dq_acc, dk_acc, dv_acc, stream); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  auto convert = [&](const float *acc, void *out, int H, const int64_t *s) {
    const uint64_t rows64 = static_cast<uint64_t>(a.B) * a.L * H;
    if (rows64 > 0xFFFFFFFFull) return cudaErrorInvalidValue;
    const uint64_t n = rows64 * (a.D / 8);
    const int blocks = static_cast<int>(n / 256 + 1 < 148 * 8 ? n / 256 + 1 : 148 * 8);
    if (a.D == 128)
      bwd_convert_kernel<128><<<blocks, 256, 0, stream>>>(acc, static_cast<__nv_bfloat16 *>(out),
                                                          static_cast<uint32_t>(rows64), H, a.L, s[0], s[1], s[2]);
    else
      bwd_convert_kernel<64><<<blocks, 256, 0, stream>>>(acc, static_cast<__nv_bfloat16 *>(out),
                                                         static_cast<uint32_t>(rows64), H, a.L, s[0], s[1], s[2]);
    return cudaGetLastError();
  };
  if ((e = convert(dq_acc, a.dq, a.Hq, a.dq_s)) != cudaSuccess) return e;
  if (tc) {
    if ((e = convert(dk_acc, a.dk, a.Hkv, a.dk_s)) != cudaSuccess) return e;
    if ((e = convert(dv_acc, a.dv, a.Hkv, a.dv_s)) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace attnsink
