// bwd_tc.cu -- backward pass of sliding-window attention with a learned
// per-head sink on the 5th-generation tensor cores (tcgen05, TMEM, TMA), head
// dimension 64 or 128.  The gradients are those of bwd.cu (page "Dao-AILab/
// flash-attention" contributor guide: the FA4 backward kernels and issue
// #2969):
//   P_ij = exp(s_ij - LSE_i), Dsum_i = dO_i . O_i,
//   dV_j = sum_i P_ij dO_i,  dS_ij = P_ij (dO_i . v_j - Dsum_i),
//   dK_j = scale sum_i dS_ij q_i,  dQ_i = scale sum_j dS_ij k_j.
// Dsum and the sink gradient come from bwd.cu's row kernel.
//
// A work unit is one block of 128 keys of one kv head (the TMEM lanes) and a
// slice of the query heads that share it; its steps walk those heads and
// every 64-query block that sees a key of the block.  Per step, five products
// with fp32 accumulators in TMEM:
//   S^T  = K Q^T      [128 keys x 64 queries]   A = K (smem), B = Q (smem)
//   dP^T = V dO^T     [128 x 64]                A = V, B = dO
//   dV  += P^T dO     [128 keys x D]            A = P^T (bf16, TMEM), B = dO (smem, N-major)
//   dK  += dS^T Q     [128 x D]                 A = dS^T (bf16, TMEM), B = Q (smem, N-major)
//   dQ^T = K^T dS^T   [128 channels x 64]       A = K (smem, M-major), B = dS^T (smem, N-major)
//                     (at D = 64 channels 64..127 are padding)
// All five have M = 128 (keys or channels on the TMEM lanes); dQ is formed
// transposed so that it needs no 64-row accumulator.  P^T and dS^T live in
// their own TMEM columns, so the next step's S^T and dP^T are computed while
// this step's exponentials are taken.  TMEM columns (512):
//   S^T 0..63 | dP^T 64..127 | P^T 128..159, dS^T 160..191 (bf16 pairs) |
//   dV 192..319 | dK 320..447 | dQ^T 448..511
//
// Warp roles (512 threads, one CTA per SM, persistent over units):
//   warps 0-7  one thread per key row and half of the step's queries (two
//              warpgroups): P^T, dS^T from S^T, dP^T, LSE, Dsum
//   warps 8-11 one thread per channel: dQ^T out of TMEM into a shared f32
//              [64 queries x 128] tile, added into the fp32 dQ workspace by
//              one TMA bulk reduction per step; at a unit's end dK, dV (rows)
//   warp 12    producer: K, V per unit, Q, dO per step (TMA, a ring of
//              kStages slots) and the step's LSE and Dsum rows
//   warp 13    TMEM allocation and the issue of S^T, dP^T (one thread)
//   warp 14    the issue of dV, dK (one thread)
//   warp 15    the issue of dQ^T (one thread): three issuers, so that no
//              group of products waits behind another's issue
// dK and dV are summed over the units of a kv head in fp32 workspaces
// (atomic adds), converted to bf16 afterwards like dQ.  Every wait is
// bounded; a timeout records ATTN_ETIMEOUT and every role returns.
#include <cuda.h>

#include <algorithm>
#include <math.h>

#include <type_traits>

#include "kernels.h"
#include "ptx.cuh"
#include "status.cuh"

namespace attnsink {
namespace {

constexpr int kBK = 128;                        // keys per unit (TMEM lanes)
constexpr int kBQ = 64;                         // queries per step
constexpr int kThreads = 512;
constexpr int kProducerWarp = 12, kMmaWarp = 13, kMmaWarp2 = 14, kMmaWarp3 = 15;
constexpr uint32_t kTmemThreads = 480;          // warps 0-11 and the three MMA warps
// Every warpgroup keeps the launch allocation (128 registers): handing some
// of the P^T/dS^T warpgroups' registers to the producer/MMA warpgroup
// measured 1-3 % slower (the exponentiation pass is latency-bound).
constexpr uint32_t kBarTmem = 1, kBarDrain = 2;
constexpr float kLog2e = 1.4426950408889634f;

constexpr uint32_t kColS = 0, kColDP = 64, kColP = 128, kColDS = 160, kTmemCols = 512;

// Pipeline depths: Q/dO ring slots (the producer runs kStages - 1 steps
// ahead), K/V buffers (2: the next unit's K, V load during this unit).
constexpr int kStages = 3, kKVBuf = 1;

constexpr int kDSTile = kBK * kBQ * 2;          // dS^T: 128 key rows of 64 queries
constexpr int kBarBytes = 256;

// Layout for head dimension D (64 or 128).  TMEM: dV and dK take D columns
// each after the fixed S^T/dP^T/P^T/dS^T columns, dQ^T 64 columns after them
// (dQ^T keeps M = 128: at D = 64 its lanes 64..127 are computed from the
// shared memory after the K tile and never read).  Shared memory, from a
// 1024-byte aligned base (128-byte swizzled tiles).
template <int D>
struct BCfg {
  static_assert(D == 64 || D == 128, "head dimension");
  static constexpr uint32_t kColDV = 192, kColDK = kColDV + D, kColDQ = kColDK + D;
  static_assert(kColDQ + kBQ <= kTmemCols, "TMEM budget");
  static constexpr int kKVTile = kBK * D * 2;           // a K or V tile: D/64 chunks of 128 rows
  static constexpr int kQTile = kBQ * D * 2;            // a Q or dO tile: D/64 chunks of 64 rows
  static constexpr int kOffK = 0;                       // [kKVBuf] K tiles
  static constexpr int kOffV = kOffK + kKVBuf * kKVTile;      // [kKVBuf] V tiles
  static constexpr int kOffQ = kOffV + kKVBuf * kKVTile;      // [kStages] Q tiles (ring slots)
  static constexpr int kOffDO = kOffQ + kStages * kQTile;     // [kStages] dO tiles
  static constexpr int kOffDS = kOffDO + kStages * kQTile;    // [2] dS^T tiles (steps alternate)
  static constexpr int kOffRow = kOffDS + 2 * kDSTile;        // [kStages][LSE*log2e x 64, Dsum x 64] f32
  static constexpr int kOffStage = kOffRow + kStages * 2 * kBQ * 4;   // dQ tile [64 queries][D] f32
  static constexpr int kOffBar = kOffStage + kBQ * D * 4;
  static constexpr int kSmemBytes = kOffBar + kBarBytes + 1024;       // + alignment slack
  static_assert(kSmemBytes <= 227 * 1024, "shared-memory budget");
  static_assert(kOffStage % 128 == 0, "bulk-copy staging alignment");
};



enum : int { kWhereKv = 201, kWhereFull = 202, kWhereEmpty = 203, kWhereS = 204, kWhereP = 205,
             kWhereDq = 206, kWhereDkv = 207 };

struct Params {
  const float *lse, *dsum;
  float *dq_acc, *dk_acc, *dv_acc;
  int *status;
  int B, L, Hq, Hkv, W, G, hsplit, nkb, num_units;
  float scale, sl2;                     // scale, scale * log2(e)
  int64_t lse_sb, lse_sh;
};

// Unit u: key block kb (slowest: the earliest blocks see the most queries
// under a causal window, so they start first), head slice hs, kv head hk,
// batch b.  Its steps are (head h0 + s / nq, query block q_lo + s % nq).
struct Unit {
  int j0, hk, b, h0, nh, q_lo, nq;
};

__device__ __forceinline__ Unit unit_at(const Params &p, int u) {
  Unit t;
  const int per_kb = p.hsplit * p.Hkv * p.B;
  const int kb = u / per_kb;
  int r = u - kb * per_kb;
  const int hs = r % p.hsplit;
  r /= p.hsplit;
  t.hk = r % p.Hkv;
  t.b = r / p.Hkv;
  t.j0 = kb * kBK;
  t.nh = p.G / p.hsplit;
  t.h0 = t.hk * p.G + hs * t.nh;
  // queries that see a key of [j0, j0 + 127]: [j0, j0 + 127 + W - 1], clipped to L
  const int last = min(p.L - 1, t.j0 + kBK - 1 + min(p.W - 1, p.L));
  t.q_lo = t.j0 / kBQ;
  t.nq = last / kBQ - t.q_lo + 1;
  return t;
}

__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, const WaitCtx &ctx, int where) {
  const bool r = mbar_wait(bar, parity, ctx, where);
  return __all_sync(0xffffffffu, r);
}

// Waits without looking at the abort flag, for draining in-flight copies on
// the way out (bounded by the same limit).
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return;
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                  const __grid_constant__ CUtensorMap tmDQ, const Params p) {
  using C = BCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *sK = smem + C::kOffK, *sV = smem + C::kOffV, *sQ = smem + C::kOffQ, *sDO = smem + C::kOffDO;
  uint8_t *sDS = smem + C::kOffDS;
  float *sRow = reinterpret_cast<float *>(smem + C::kOffRow);
  uint64_t *kv_full = reinterpret_cast<uint64_t *>(smem + C::kOffBar);   // [kKVBuf] K, V of a unit landed
  uint64_t *kv_empty = kv_full + kKVBuf; // [kKVBuf] a unit's last product read its K, V
  uint64_t *full = kv_empty + kKVBuf;    // [kStages] a step's Q, dO (TMA) and rows (32 lanes) landed
  uint64_t *empty = full + kStages;      // [kStages] a step's dV, dK products read its Q, dO
  uint64_t *s_full = empty + kStages;    // S^T, dP^T of a step computed
  uint64_t *s_free = s_full + 1;         // ... and read out of TMEM (256 arrivals)
  uint64_t *p_full = s_free + 1;         // P^T, dS^T of a step in TMEM and dS^T in smem (256)
  uint64_t *pbuf_free = p_full + 1;      // a step's dV, dK products read P^T, dS^T
  uint64_t *dq_full = pbuf_free + 1;     // a step's dQ^T computed
  uint64_t *dq_empty = dq_full + 1;      // ... and read out of TMEM (128)
  uint64_t *dsm_free = dq_empty + 1;     // [2] a step's dQ^T product read its dS^T tile
  uint64_t *dkv_full = dsm_free + 2;     // a unit's last dV, dK products finished
  uint64_t *dkv_free = dkv_full + 1;     // ... and dK, dV read out of TMEM (128)
  uint64_t *mma_done = dkv_free + 1;     // every product of the CTA finished (all three issuers)
  // [2] dS^T of step g in shared memory (256), for the dQ^T issuer: one per
  // dS^T buffer, so that each advances once every two steps and the softmax,
  // which the dS^T buffers let run at most two steps ahead of that issuer,
  // cannot bring a barrier back to the parity it waits for
  uint64_t *dsp_full = mma_done + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(dsp_full + 2);
  int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
  const WaitCtx ctx{abort_flag, p.status, wait_limit_ns(p.status)};

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kKVBuf; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 32);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) mbar_init(&dsm_free[i], 1);
    mbar_init(s_full, 1);
    mbar_init(s_free, 256);
    mbar_init(p_full, 256);
    mbar_init(pbuf_free, 1);
    mbar_init(dq_full, 1);
    mbar_init(dq_empty, 128);
    mbar_init(dkv_full, 1);
    mbar_init(dkv_free, 128);
    mbar_init(mma_done, 3);
    for (int i = 0; i < 2; ++i) mbar_init(&dsp_full[i], 256);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // TMEM: the MMA warp allocates all 512 columns (one CTA per SM); the TMEM
  // warps read the base after one named barrier of exactly those warps.
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  uint32_t tmem = 0;
  const bool tmem_warp = warp < 12 || warp == kMmaWarp || warp == kMmaWarp2 || warp == kMmaWarp3;
  if (tmem_warp) {
    tc_fence_before();
    named_barrier_sync(kBarTmem, kTmemThreads);
    tc_fence_after();
    tmem = *tmem_slot;
  }
  if (warp >= 12) {
  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
    }
    bool ok = true;
    int g = 0, ul = 0;
    int kv_issued = 0;                        // units whose K, V copies were issued
    for (int u = blockIdx.x; ok && u < p.num_units; u += gridDim.x, ++ul) {
      const Unit t = unit_at(p, u);
      const int kvb = ul % kKVBuf;
      if (lane == 0) {
        // the buffer's previous unit has finished with its K and V
        if (ul >= kKVBuf &&
            !mbar_wait(&kv_empty[kvb], static_cast<uint32_t>(ul / kKVBuf - 1) & 1u, ctx, kWhereKv))
          ok = false;
        if (ok) {
          mbar_arrive_expect_tx(&kv_full[kvb], 2 * C::kKVTile);
          for (int c = 0; c < D / 64; ++c) {
            tma_load_4d(sK + kvb * C::kKVTile + c * kBK * 128, &tmK, &kv_full[kvb], c * 64, t.hk, t.j0, t.b);
            tma_load_4d(sV + kvb * C::kKVTile + c * kBK * 128, &tmV, &kv_full[kvb], c * 64, t.hk, t.j0, t.b);
          }
          kv_issued = ul + 1;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      const int steps = t.nh * t.nq;
      for (int s = 0; ok && s < steps; ++s) {
        const int slot = g % kStages;
        const int h = t.h0 + s / t.nq;
        const int i0 = (t.q_lo + s % t.nq) * kBQ;
        // the step's rows, fetched while the slot drains: LSE in log2 units
        // (+inf past the end, so P = 0) and Dsum
        float lr[kBQ / 32], dr[kBQ / 32];
#pragma unroll
        for (int e = 0; e < kBQ / 32; ++e) {
          const int i = i0 + lane + 32 * e;
          const bool in = i < p.L;
          lr[e] = in ? p.lse[t.b * p.lse_sb + h * p.lse_sh + i] * kLog2e : INFINITY;
          dr[e] = in ? p.dsum[(static_cast<int64_t>(t.b) * p.Hq + h) * p.L + i] : 0.f;
        }
        if (lane == 0 && g >= kStages &&
            !mbar_wait(&empty[slot], static_cast<uint32_t>(g / kStages - 1) & 1u, ctx, kWhereEmpty))
          ok = false;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        float *row = sRow + slot * 2 * kBQ;
#pragma unroll
        for (int e = 0; e < kBQ / 32; ++e) {
          row[lane + 32 * e] = lr[e];
          row[kBQ + lane + 32 * e] = dr[e];
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[slot], 2 * C::kQTile);
          for (int c = 0; c < D / 64; ++c) {
            tma_load_4d(sQ + slot * C::kQTile + c * kBQ * 128, &tmQ, &full[slot], c * 64, h, i0, t.b);
            tma_load_4d(sDO + slot * C::kQTile + c * kBQ * 128, &tmDO, &full[slot], c * 64, h, i0, t.b);
          }
        } else {
          mbar_arrive(&full[slot]);
        }
        ++g;                                  // steps whose copies were issued
      }
    }
    if (lane == 0) {
      // Before this warp leaves, the copies it issued have landed: the CTA
      // (and its shared memory) must outlive them even when the other roles
      // gave up early.  In a normal run they are long done.
      for (int k = max(0, kv_issued - kKVBuf); k < kv_issued; ++k)
        drain_wait(&kv_full[k % kKVBuf], static_cast<uint32_t>(k / kKVBuf) & 1u);
      for (int k = max(0, g - kStages); k < g; ++k)
        drain_wait(&full[k % kStages], static_cast<uint32_t>(k / kStages) & 1u);
    }
    __syncwarp();
  } else if (warp == kMmaWarp || warp == kMmaWarp2 || warp == kMmaWarp3) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idesc_s = umma_idesc_bf16(kBK, kBQ, 0, 0);    // K-major A and B
      constexpr uint32_t idesc_kv = umma_idesc_bf16(kBK, D, 0, 1);    // A in TMEM, B N-major
      constexpr uint32_t idesc_dq = umma_idesc_bf16(128, kBQ, 1, 1);  // A M-major (M = 128 >= D), B N-major
      // 128-byte swizzle, 8-row groups 1024 bytes apart; the leading offset is
      // the distance between 64-element chunks along M or N for the
      // M/N-major operands (K-major operands ignore it)
      const uint32_t hi = umma_desc_hi_sw128(1024);
      const uint32_t k_lo = umma_desc_lo(smem_u32(sK), 16);
      const uint32_t v_lo = umma_desc_lo(smem_u32(sV), 16);
      const uint32_t q_lo = umma_desc_lo(smem_u32(sQ), 16);
      const uint32_t do_lo = umma_desc_lo(smem_u32(sDO), 16);
      const uint32_t qn_lo = umma_desc_lo(smem_u32(sQ), kBQ * 128);     // Q as an N-major B
      const uint32_t don_lo = umma_desc_lo(smem_u32(sDO), kBQ * 128);   // dO as an N-major B
      const uint32_t km_lo = umma_desc_lo(smem_u32(sK), kBK * 128);     // K as an M-major A
      const uint32_t ds_lo = umma_desc_lo(smem_u32(sDS), kBK * 128);    // dS^T as an N-major B
      bool ok = true;
      int g = 0, ul = 0;
      if (warp == kMmaWarp) {
        // S^T = K Q^T and dP^T = V dO^T per step, once the softmax warps have
        // read the previous step's out of TMEM
        for (int u = blockIdx.x; ok && u < p.num_units; u += gridDim.x, ++ul) {
          const Unit t = unit_at(p, u);
          const int kvb = ul % kKVBuf;
          if (!mbar_wait(&kv_full[kvb], static_cast<uint32_t>(ul / kKVBuf) & 1u, ctx, kWhereKv)) {
            ok = false;
            break;
          }
          const int steps = t.nh * t.nq;
          for (int s = 0; s < steps; ++s, ++g) {
            const int slot = g % kStages;
            if (!mbar_wait(&full[slot], static_cast<uint32_t>(g / kStages) & 1u, ctx, kWhereFull)) {
              ok = false;
              break;
            }
            if (g > 0 && !mbar_wait(s_free, static_cast<uint32_t>(g - 1) & 1u, ctx, kWhereS)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              // 16 channels = 32 bytes along the swizzled row; 64-channel chunks apart
              const uint32_t ka = ((kvb * C::kKVTile + (kk >> 2) * kBK * 128) >> 4) + (kk & 3) * 2;
              const uint32_t qa = ((slot * C::kQTile + (kk >> 2) * kBQ * 128) >> 4) + (kk & 3) * 2;
              umma_ss_w(tmem + kColS, k_lo + ka, hi, q_lo + qa, hi, idesc_s, kk > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t ka = ((kvb * C::kKVTile + (kk >> 2) * kBK * 128) >> 4) + (kk & 3) * 2;
              const uint32_t qa = ((slot * C::kQTile + (kk >> 2) * kBQ * 128) >> 4) + (kk & 3) * 2;
              umma_ss_w(tmem + kColDP, v_lo + ka, hi, do_lo + qa, hi, idesc_s, kk > 0 ? 1u : 0u);
            }
            umma_commit(s_full);
          }
        }
      } else if (warp == kMmaWarp2) {
        // dV += P^T dO and dK += dS^T Q once P^T, dS^T of the step are in.
        // (The step's Q, dO landed before the S^T product that led to P^T;
        // the wait below is already complete and only orders this thread
        // after the copies.  The S^T, dP^T products that read the slot
        // finished before the softmax read S^T, so the release committed here
        // follows them.)
        for (int u = blockIdx.x; ok && u < p.num_units; u += gridDim.x, ++ul) {
          const Unit t = unit_at(p, u);
          const int steps = t.nh * t.nq;
          for (int s = 0; s < steps; ++s, ++g) {
            const int slot = g % kStages;
            const bool first = s == 0, last = s == steps - 1;
            if (!mbar_wait(p_full, static_cast<uint32_t>(g) & 1u, ctx, kWhereP) ||
                !mbar_wait(&full[slot], static_cast<uint32_t>(g / kStages) & 1u, ctx, kWhereFull)) {
              ok = false;
              break;
            }
            // the first step of a unit overwrites dK, dV: the previous unit's
            // must have been read out of TMEM
            if (first && ul > 0 && !mbar_wait(dkv_free, static_cast<uint32_t>(ul - 1) & 1u, ctx, kWhereDkv)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t acc0 = first ? 0u : 1u;
#pragma unroll
            for (int kk = 0; kk < kBQ / 16; ++kk)
              umma_ts_w(tmem + C::kColDV, tmem + kColP + kk * 8, don_lo + ((slot * C::kQTile + kk * 16 * 128) >> 4),
                        hi, idesc_kv, kk > 0 ? 1u : acc0);
#pragma unroll
            for (int kk = 0; kk < kBQ / 16; ++kk)
              umma_ts_w(tmem + C::kColDK, tmem + kColDS + kk * 8, qn_lo + ((slot * C::kQTile + kk * 16 * 128) >> 4),
                        hi, idesc_kv, kk > 0 ? 1u : acc0);
            umma_commit(pbuf_free);
            umma_commit(&empty[slot]);
            if (last) umma_commit(dkv_full);
          }
        }
      } else {
        // dQ^T = K^T dS^T once dS^T of the step is in shared memory and the
        // previous dQ^T has been read out.  (The unit's K landed before its
        // first S^T product; the K/V release committed here at a unit's end
        // follows that unit's S^T, dP^T products, which finished before the
        // softmax read them.)
        for (int u = blockIdx.x; ok && u < p.num_units; u += gridDim.x, ++ul) {
          const Unit t = unit_at(p, u);
          const int kvb = ul % kKVBuf;
          const int steps = t.nh * t.nq;
          for (int s = 0; s < steps; ++s, ++g) {
            const bool first = s == 0, last = s == steps - 1;
            if (!mbar_wait(&dsp_full[g & 1], static_cast<uint32_t>(g >> 1) & 1u, ctx, kWhereP) ||
                (first && !mbar_wait(&kv_full[kvb], static_cast<uint32_t>(ul / kKVBuf) & 1u, ctx, kWhereKv)) ||
                (g > 0 && !mbar_wait(dq_empty, static_cast<uint32_t>(g - 1) & 1u, ctx, kWhereDq))) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk)
              umma_ss_w(tmem + C::kColDQ, km_lo + ((kvb * C::kKVTile + kk * 16 * 128) >> 4), hi,
                        ds_lo + (((g & 1) * kDSTile + kk * 16 * 128) >> 4), hi, idesc_dq, kk > 0 ? 1u : 0u);
            umma_commit(dq_full);
            umma_commit(&dsm_free[g & 1]);
            if (last) umma_commit(&kv_empty[kvb]);
          }
        }
      }
      // Every tensor-core operation of this CTA has finished before teardown
      // (every issuer arrives).
      umma_commit(mma_done);
      drain_wait(mma_done, 0);
    }
    __syncwarp();
  }
  } else if (warp < 8) {
    // --------------- P^T, dS^T: one key row per thread, 32 query columns per
    // warpgroup (warpgroup 0 the first half of the step's queries)
    const int r = threadIdx.x & 127;                  // key row == TMEM lane
    const int c0 = (warp >> 2) * 32;                  // this warpgroup's first column
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    bool ok = true;
    int g = 0;
    for (int u = blockIdx.x; ok && u < p.num_units; u += gridDim.x) {
      const Unit t = unit_at(p, u);
      const int j = t.j0 + r;                         // key position
      const int steps = t.nh * t.nq;
      for (int s = 0; s < steps; ++s, ++g) {
        const int slot = g % kStages;
        const int i0 = (t.q_lo + s % t.nq) * kBQ;
        if (!warp_wait(s_full, static_cast<uint32_t>(g) & 1u, ctx, kWhereS) ||
            !warp_wait(&full[slot], static_cast<uint32_t>(g / kStages) & 1u, ctx, kWhereFull)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sv[32], dv[32];
        tmem_ld32(lane_base + kColS + c0, sv);
        tmem_ld32(lane_base + kColDP + c0, dv);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(s_free);                          // the next step's S^T, dP^T may start
        // Does any (key, query) pair of the step fall outside the window or
        // past the end of the sequence?  If so, this row's visible columns
        // are [vlo, vhi] (query i = i0 + column sees key j iff
        // j <= i < L and i - j < W).
        const bool edge = (t.j0 + kBK - 1 > i0) || (t.j0 < i0 + kBQ - p.W) || (i0 + kBQ > p.L);
        const int vlo = j - i0;
        const int vhi = min(j - i0 + min(p.W - 1, p.L), p.L - 1 - i0);
        const float4 *lse4 = reinterpret_cast<const float4 *>(sRow + slot * 2 * kBQ + c0);
        const float4 *dsum4 = lse4 + kBQ / 4;
        uint32_t pp[16], dd[16];                      // bf16 pairs of P^T and dS^T
        // one branch-free copy per case (a per-element branch inside the
        // unrolled loop costs the unmasked steps as much as the masked ones)
        auto cols = [&](auto masked) {
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            const float4 l4 = lse4[c >> 2];
            const float4 m4 = dsum4[c >> 2];
            const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
            const float mv[4] = {m4.x, m4.y, m4.z, m4.w};
            float pe[4], de[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              pe[e] = ex2_approx(__uint_as_float(sv[c + e]) * p.sl2 - lv[e]);
              if constexpr (decltype(masked)::value) {
                const int col = c0 + c + e;
                pe[e] = (col >= vlo && col <= vhi) ? pe[e] : 0.f;
              }
              de[e] = pe[e] * (__uint_as_float(dv[c + e]) - mv[e]);
            }
            pp[c / 2] = pack_bf16x2(pe[0], pe[1]);
            pp[c / 2 + 1] = pack_bf16x2(pe[2], pe[3]);
            dd[c / 2] = pack_bf16x2(de[0], de[1]);
            dd[c / 2 + 1] = pack_bf16x2(de[2], de[3]);
          }
        };
        if (edge)
          cols(std::true_type{});
        else
          cols(std::false_type{});
        // P^T, dS^T overwrite the previous step's (its dV, dK products must
        // have read them); dS^T's shared tile was last read two steps ago
        if ((g > 0 && !warp_wait(pbuf_free, static_cast<uint32_t>(g - 1) & 1u, ctx, kWhereP)) ||
            (g >= 2 && !warp_wait(&dsm_free[g & 1], static_cast<uint32_t>((g >> 1) - 1) & 1u, ctx, kWhereDq))) {
          ok = false;
          break;
        }
        tc_fence_after();
        tmem_st16(lane_base + kColP + c0 / 2, pp);
        tmem_st16(lane_base + kColDS + c0 / 2, dd);
        // dS^T row r: 64 queries = 128 bytes, 16-byte units swizzled by row;
        // this warpgroup's 32 queries are units c0/8 .. c0/8 + 3
        uint8_t *dsrow = sDS + (g & 1) * kDSTile + r * 128;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4 *>(dsrow + (((c0 / 8 + q) ^ (r & 7)) << 4)) =
              make_uint4(dd[4 * q], dd[4 * q + 1], dd[4 * q + 2], dd[4 * q + 3]);
        tmem_wait_st();
        fence_proxy_async_smem();                     // dS^T visible to the tensor cores
        tc_fence_before();
        mbar_arrive(p_full);
        mbar_arrive(&dsp_full[g & 1]);
      }
    }
  } else {
    // ------------------------- dQ^T out of TMEM; dK, dV at the end of a unit
    const int rr = (warp & 3) * 32 + lane;            // TMEM lane: channel (dQ^T), key row (dK, dV)
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    float *stage = reinterpret_cast<float *>(smem + C::kOffStage);
    bool ok = true;
    int g = 0, ul = 0;
    for (int u = blockIdx.x; ok && u < p.num_units; u += gridDim.x, ++ul) {
      const Unit t = unit_at(p, u);
      const int steps = t.nh * t.nq;
      for (int s = 0; s < steps; ++s, ++g) {
        const int h = t.h0 + s / t.nq;
        const int i0 = (t.q_lo + s % t.nq) * kBQ;
        // the previous step's reduction has read the staging tile
        if (rr == 0) tma_store_wait_read();
        // The four warps' vote (the barrier that also publishes the read
        // above): they go on, or leave, together, so the barrier below is
        // met by all of them.
        const bool got = warp_wait(dq_full, static_cast<uint32_t>(g) & 1u, ctx, kWhereDq);
        if (!named_barrier_and(kBarDrain, 128, got)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t x0[32], x1[32];
        tmem_ld32(lane_base + C::kColDQ, x0);
        tmem_ld32(lane_base + C::kColDQ + 32, x1);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(dq_empty);                        // the next dQ^T may overwrite it
        // dQ^T column -> dQ row-major tile: for each query the warp writes 32
        // consecutive channels
        if (rr < D) {                                 // (lanes past D hold padding)
#pragma unroll
          for (int c = 0; c < 32; ++c) stage[c * D + rr] = __uint_as_float(x0[c]) * p.scale;
#pragma unroll
          for (int c = 0; c < 32; ++c) stage[(32 + c) * D + rr] = __uint_as_float(x1[c]) * p.scale;
        }
        fence_proxy_async_smem();
        named_barrier_sync(kBarDrain, 128);
        if (rr == 0) {
          // rows past the end of the sequence are clipped by the unit
          tma_reduce_add_4d(&tmDQ, stage, 0, h, i0, t.b);
          tma_store_commit();
        }
        if (s == steps - 1) {
          const bool kv_ok = warp_wait(dkv_full, static_cast<uint32_t>(ul) & 1u, ctx, kWhereDkv);
          if (!named_barrier_and(kBarDrain, 128, kv_ok)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int j = t.j0 + rr;
          const int64_t kv_row = ((static_cast<int64_t>(t.b) * p.L + j) * p.Hkv + t.hk) * D;
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t k32[32], v32[32];
            tmem_ld32(lane_base + C::kColDK + c * 32, k32);
            tmem_ld32(lane_base + C::kColDV + c * 32, v32);
            tmem_wait_ld();
            if (j < p.L) {
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                atomicAdd(reinterpret_cast<float4 *>(p.dk_acc + kv_row + c * 32 + 4 * q),
                          make_float4(__uint_as_float(k32[4 * q]) * p.scale, __uint_as_float(k32[4 * q + 1]) * p.scale,
                                      __uint_as_float(k32[4 * q + 2]) * p.scale, __uint_as_float(k32[4 * q + 3]) * p.scale));
                atomicAdd(reinterpret_cast<float4 *>(p.dv_acc + kv_row + c * 32 + 4 * q),
                          make_float4(__uint_as_float(v32[4 * q]), __uint_as_float(v32[4 * q + 1]),
                                      __uint_as_float(v32[4 * q + 2]), __uint_as_float(v32[4 * q + 3])));
              }
            }
          }
          tc_fence_before();
          mbar_arrive(dkv_free);                      // the next unit's first dV, dK may overwrite them
        }
      }
    }
    // the reductions must have read shared memory before the CTA leaves
    if (rr == 0) tma_store_wait_all();
  }
  // ---- teardown: every TMEM user is done before the allocator frees it ----
  if (tmem_warp) {
    tc_fence_before();
    named_barrier_sync(kBarTmem, kTmemThreads);
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
cudaError_t launch_tc(const BwdArgs &a, const float *dsum, float *dq_acc, float *dk_acc, float *dv_acc,
                      cudaStream_t stream) {
  using C = BCfg<D>;
  alignas(64) CUtensorMap mq, mk, mv, mdo, mdq;
  cudaError_t e;
  if ((e = make_tma_bshd(&mq, a.q, a.B, a.L, a.Hq, D, a.q_s, kBQ)) != cudaSuccess) return e;
  if ((e = make_tma_bshd(&mk, a.k, a.B, a.L, a.Hkv, D, a.k_s, kBK)) != cudaSuccess) return e;
  if ((e = make_tma_bshd(&mv, a.v, a.B, a.L, a.Hkv, D, a.v_s, kBK)) != cudaSuccess) return e;
  if ((e = make_tma_bshd(&mdo, a.dout, a.B, a.L, a.Hq, D, a.do_s, kBQ)) != cudaSuccess) return e;
  const int64_t acc_s[3] = {static_cast<int64_t>(a.L) * a.Hq * D, static_cast<int64_t>(a.Hq) * D, D};
  if ((e = make_tma_bshd(&mdq, dq_acc, a.B, a.L, a.Hq, D, acc_s, kBQ, 4)) != cudaSuccess) return e;
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  static int sm_count[64] = {};
  if (dev >= 0 && dev < 64 && sm_count[dev] == 0)
    if ((e = cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return e;
  const int sms = (dev >= 0 && dev < 64) ? sm_count[dev] : 148;
  Params p;
  p.lse = a.lse;
  p.dsum = dsum;
  p.dq_acc = dq_acc;
  p.dk_acc = dk_acc;
  p.dv_acc = dv_acc;
  p.status = a.status;
  p.B = a.B;
  p.L = a.L;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.W = a.W;
  p.G = a.Hq / a.Hkv;
  p.nkb = (a.L + kBK - 1) / kBK;
  // Split each kv head's query heads over units (whole heads per unit; the
  // units of a kv head add their dK, dV into the same fp32 rows): the fewest
  // units whose largest is at most a fifth of an SM's average share of the
  // steps.  The static schedule then ends within about that of the average,
  // and every further unit costs a K/V load and a dK/dV write-out.  A key
  // block kb sees query blocks 2 kb .. last(kb) / 64, last(kb) =
  // min(L - 1, 128 kb + 127 + min(W - 1, L)); block 0 sees the most.
  const int64_t base = static_cast<int64_t>(p.nkb) * a.Hkv * a.B;
  const int64_t wc = a.W - 1 < a.L ? a.W - 1 : a.L;
  const int64_t nq_int = (127 + wc) / 64 + 1;               // blocks whose window ends before L - 1
  const int64_t k1 = a.L - 1 - 127 - wc >= 0
                         ? std::min<int64_t>(p.nkb, (a.L - 1 - 127 - wc) / 128 + 1) : 0;
  const int64_t qlast = (a.L - 1) / 64, ntail = p.nkb - k1;
  const int64_t steps_per_head = k1 * nq_int + ntail * (qlast + 1) - (k1 + p.nkb - 1) * ntail;
  const int64_t nq_max = std::min<int64_t>(a.L - 1, 127 + wc) / 64 + 1;
  const int64_t total_steps = steps_per_head * a.Hq * a.B;
  p.hsplit = p.G;
  for (int hs = 1; hs <= p.G; ++hs) {
    if (p.G % hs) continue;
    if (base * hs >= sms && 5 * (p.G / hs) * nq_max * sms <= total_steps) {
      p.hsplit = hs;
      break;
    }
  }
  const int64_t units = base * p.hsplit;
  if (units > (1LL << 30)) return cudaErrorInvalidValue;
  p.num_units = static_cast<int>(units);
  p.scale = a.scale;
  p.sl2 = static_cast<float>(static_cast<double>(a.scale) * 1.4426950408889634);
  p.lse_sb = a.lse_s[0];
  p.lse_sh = a.lse_s[1];
  if ((e = cudaFuncSetAttribute(bwd_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes)) !=
      cudaSuccess)
    return e;
  const int grid = static_cast<int>(units < sms ? units : sms);
  bwd_tc_kernel<D><<<grid, kThreads, C::kSmemBytes, stream>>>(mq, mk, mv, mdo, mdq, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_main_tc(const BwdArgs &a, const float *dsum, float *dq_acc, float *dk_acc, float *dv_acc,
                               cudaStream_t stream) {
  switch (a.D) {
    case 64: return launch_tc<64>(a, dsum, dq_acc, dk_acc, dv_acc, stream);
    case 128: return launch_tc<128>(a, dsum, dq_acc, dk_acc, dv_acc, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace attnsink
