// fwd_tc.cu -- prefill forward of sliding-window attention with a learned
// per-head sink on the Blackwell tensor cores (tcgen05 + TMEM + TMA).
//
// Method: page "cf-1.com/news/6055759" (Flint's learned sink, W = 513):
// softmax over the W most recent keys plus one sink logit per head in the
// denominator; its "fix 2" gives the epilogue (rebase the running maximum on
// the sink, rescale the denominator and the output by the same factor) and
// its "fix 1" the rule for the TMEM allocation barrier (every warp that uses
// TMEM takes part in it, and one constant defines that set).  The kernel
// layout follows the FA4 SM100 design the flash-attention contributor-guide
// page describes (load / MMA / softmax roles, S and O accumulated in TMEM) as
// prior art; everything here is written for sm_100a directly.
//
// One CTA computes one 128-row query tile of one head:
//   warp 4      TMA producer: Q once, then K/V tiles into a ring of stages in
//               the order the MMA warp consumes them (K0, K1, V0, K2, V1, ...)
//   warp 5      TMEM allocator and MMA issuer: S_j = Q K_j^T into one of two
//               TMEM S buffers, O += P_j V_j with P_j read from TMEM
//   warps 0-3   softmax / correction / epilogue, one thread per query row
//               (TMEM lane); P_j is written as bf16 over S_j's columns.
// Only the K tiles that meet the window [m0-W+1, m0+127] are visited; the
// mask is applied on the tiles that cross the causal diagonal, the window's
// lower edge or the end of the sequence.
#include <math.h>

#include "kernels.h"
#include "ptx.cuh"

namespace attnsink {
namespace {

constexpr int kBM = 128;             // query rows per tile (= TMEM lanes)
constexpr int kSoftmaxWarps = 4;     // warps 0..3
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kThreads = 6 * 32;
// The warps that touch TMEM: the softmax warpgroup and the MMA warp.  This is
// the single definition of the TMEM allocation barrier's participant set; the
// barrier count and the participation test below both derive from it.
constexpr uint32_t kTmemWarpMask = 0x0Fu | (1u << kMmaWarp);
constexpr uint32_t kTmemThreads = 32u * __builtin_popcount(kTmemWarpMask);
__host__ __device__ constexpr bool is_tmem_warp(int w) { return (kTmemWarpMask >> w) & 1u; }

constexpr uint32_t kBarTmem = 1;     // named barrier ids (0 = __syncthreads)
constexpr uint32_t kBarEpilogue = 2;
constexpr uint32_t kTmemCols = 512;
// Lazy rescaling: the running maximum (log2 units) only moves when a tile's
// maximum exceeds it by more than this; until then exponents stay <= 2^8.
constexpr float kRescaleThreshold = 8.0f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// wait-location codes reported with ATTN_ETIMEOUT
enum : int { kWhereQ = 101, kWhereFull = 102, kWhereEmpty = 103, kWhereS = 104, kWhereP = 105,
             kWhereO = 106 };

template <int D, int BN>
struct Cfg {
  static constexpr int kChunks = D / 64;          // 64-channel (128-byte) column chunks
  static constexpr int kQBytes = kBM * D * 2;
  static constexpr int kTileBytes = BN * D * 2;   // one K or V tile
  static constexpr int kStages = (D == 64) ? 8 : (D == 128 ? 5 : 4);
  static constexpr int kRingBytes = kStages * kTileBytes;
  static constexpr int kBarOffset = kQBytes + kRingBytes;
  static constexpr int kSmemBytes = kBarOffset + 256 + 1024;  // + barriers + alignment slack
  static constexpr uint32_t kOCol = 2 * BN;                    // O accumulator column
  static_assert(2 * BN + D <= (int)kTmemCols, "TMEM budget");
  static_assert(kSmemBytes <= 227 * 1024, "shared-memory budget");
};

struct Params {
  int L, Hq, W, group, num_m_tiles;
  float scale_log2;
  const float *sinks;
  float *lse;
  int64_t lse_sb, lse_sh;
  int *status;
};

// Warp-uniform bounded wait: every lane learns the same outcome, so the
// .sync.aligned tcgen05 instructions that follow stay convergent.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, const WaitCtx &ctx,
                                          int where) {
  const bool r = mbar_wait(bar, parity, ctx, where);
  return __all_sync(0xffffffffu, r);
}

// Wait without looking at the abort flag, for draining in-flight async work
// on the way out (bounded by the same limit).
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return;
  }
}

template <int D, int BN>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                  const Params p) {
  using C = Cfg<D, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *sQ = smem;                       // Q tile, later the O staging tile
  uint8_t *sRing = smem + C::kQBytes;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarOffset);
  uint64_t *empty = full + C::kStages;
  uint64_t *q_full = empty + C::kStages;
  uint64_t *s_full = q_full + 1;            // [2]
  uint64_t *p_full = s_full + 2;
  uint64_t *o_full = p_full + 1;
  uint64_t *mma_done = o_full + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
  int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
  const WaitCtx ctx{abort_flag, p.status};

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Later query tiles see more keys under a causal window; launch them first.
  const int mt = p.num_m_tiles - 1 - static_cast<int>(blockIdx.x);
  const int h = blockIdx.y, b = blockIdx.z;
  const int hk = h / p.group;
  const int m0 = mt * kBM;
  const int row_last = min(p.L - 1, m0 + kBM - 1);
  const int key_lo = max(0, m0 - p.W + 1);
  const int kt0 = key_lo / BN;
  const int n_tiles = row_last / BN - kt0 + 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(p_full, kSoftmaxWarps * 32);
    mbar_init(o_full, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  // ---- TMEM allocation (page "cf-1.com/news/6055759", fix 1) ----
  // The MMA warp allocates; every TMEM warp then meets at one named barrier
  // whose count is exactly the number of threads in kTmemWarpMask, and only
  // after it reads the column base.
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  uint32_t tmem = 0;
  if (is_tmem_warp(warp)) {
    tc_fence_before();
    named_barrier_sync(kBarTmem, kTmemThreads);
    tc_fence_after();
    tmem = *tmem_slot;
  }

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(q_full, C::kQBytes);
      for (int c = 0; c < C::kChunks; ++c)
        tma_load_4d(sQ + c * kBM * 128, &tmQ, q_full, c * 64, h, m0, b);
      int slot = 0;
      bool ok = true;
      auto load = [&](const CUtensorMap *map, int kt) {
        const int s = slot % C::kStages;
        const uint32_t use = static_cast<uint32_t>(slot / C::kStages);
        if (slot >= C::kStages && !mbar_wait(&empty[s], (use & 1u) ^ 1u, ctx, kWhereEmpty)) {
          ok = false;
          return;
        }
        mbar_arrive_expect_tx(&full[s], C::kTileBytes);
        uint8_t *dst = sRing + s * C::kTileBytes;
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_4d(dst + c * BN * 128, map, &full[s], c * 64, hk, kt * BN, b);
        ++slot;
      };
      load(&tmK, kt0);
      for (int j = 0; ok && j < n_tiles; ++j) {
        if (j + 1 < n_tiles) load(&tmK, kt0 + j + 1);
        if (ok) load(&tmV, kt0 + j);
      }
      if (!ok) {
        // Leaving early: let the copies already issued land before the CTA
        // (and its shared memory) goes away.
        drain_wait(q_full, 0);
        for (int t = max(0, slot - C::kStages); t < slot; ++t)
          drain_wait(&full[t % C::kStages], static_cast<uint32_t>(t / C::kStages) & 1u);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idesc_qk = umma_idesc_bf16(kBM, BN, 0, 0);  // Q, K both K-major
      constexpr uint32_t idesc_pv = umma_idesc_bf16(kBM, D, 0, 1);   // V is N-major
      const uint32_t q_base = smem_u32(sQ);
      const uint32_t ring_base = smem_u32(sRing);
      bool ok = mbar_wait(q_full, 0, ctx, kWhereQ);
      int slot = 0;
      auto acquire = [&](int &s) {
        s = slot % C::kStages;
        ok = ok && mbar_wait(&full[s], static_cast<uint32_t>(slot / C::kStages) & 1u, ctx,
                             kWhereFull);
        ++slot;
        tc_fence_after();
        return ok;
      };
      auto issue_s = [&](int j, int s) {
        const uint32_t d_tmem = tmem + static_cast<uint32_t>((j & 1) * BN);
        const uint32_t k_base = ring_base + s * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk & 3) * 32;   // 16 channels = 32 bytes along the row
          const uint64_t a = umma_smem_desc_sw128(q_base + (kk >> 2) * (kBM * 128) + koff, 16, 1024);
          const uint64_t bd = umma_smem_desc_sw128(k_base + (kk >> 2) * (BN * 128) + koff, 16, 1024);
          umma_ss(d_tmem, a, bd, idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[j & 1]);
        umma_commit(&empty[s]);
      };
      auto issue_pv = [&](int j, int s) {
        const uint32_t a_tmem = tmem + static_cast<uint32_t>((j & 1) * BN);
        const uint32_t v_base = ring_base + s * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t bd = umma_smem_desc_sw128(v_base + kk * 16 * 128, BN * 128, 1024);
          umma_ts(tmem + C::kOCol, a_tmem + kk * 8, bd, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(o_full);
        umma_commit(&empty[s]);
      };
      int s;
      if (ok && acquire(s)) issue_s(0, s);
      for (int j = 0; ok && j < n_tiles; ++j) {
        if (j + 1 < n_tiles) {
          if (!acquire(s)) break;
          issue_s(j + 1, s);
        }
        if (!mbar_wait(p_full, static_cast<uint32_t>(j) & 1u, ctx, kWhereP)) break;
        tc_fence_after();
        if (!acquire(s)) break;
        issue_pv(j, s);
      }
      // Every tensor-core operation of this CTA has finished before teardown.
      umma_commit(mma_done);
      drain_wait(mma_done, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------- softmax / correction / epilogue
    const int r = threadIdx.x;                       // tile row == TMEM lane
    const int i = m0 + r;                            // query position
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY;                         // running max, log2 units
    float l_run = 0.f;                               // running denominator
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      if (!warp_wait(&s_full[j & 1], static_cast<uint32_t>(j >> 1) & 1u, ctx, kWhereS)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t s_addr = lane_base + static_cast<uint32_t>((j & 1) * BN);
      float s[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t raw[32];
        tmem_ld32(s_addr + c * 32, raw);
        tmem_wait_ld();
#pragma unroll
        for (int t = 0; t < 32; ++t) s[c * 32 + t] = __uint_as_float(raw[t]);
      }
      const int kbase = (kt0 + j) * BN;
      // Tile-uniform test: does any (row, key) of this tile fall outside the
      // causal window or past the end of the sequence?
      const bool edge = (kbase + BN - 1 > m0) || (kbase < m0 + kBM - p.W) || (kbase + BN > p.L);
      if (edge) {
        const int lo = i - p.W + 1 - kbase;          // first visible column
        const int hi = min(i, p.L - 1) - kbase;      // last visible column
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (c < lo || c > hi) s[c] = -INFINITY;
      }
      float mt = s[0];
#pragma unroll
      for (int c = 1; c < BN; ++c) mt = fmaxf(mt, s[c]);
      const float mt2 = mt * sl2;
      float alpha = 1.f;
      if (mt2 > m_run + kRescaleThreshold) {
        alpha = ex2_approx(m_run - mt2);             // 0 while nothing was seen yet
        m_run = mt2;
      }
      l_run *= alpha;
      if (j > 0) {
        // O holds sum_{t<j} P_t V_t: wait for PV_{j-1}, then rescale it if
        // any row of this warp moved its maximum.
        if (!warp_wait(o_full, static_cast<uint32_t>(j - 1) & 1u, ctx, kWhereO)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(lane_base + C::kOCol + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int t = 0; t < 32; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * alpha);
            tmem_st32(lane_base + C::kOCol + c * 32, o);
          }
        }
      }
      const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          const float p0 = ex2_approx(fmaf(s[c * 32 + 2 * t], sl2, -m_use));
          const float p1 = ex2_approx(fmaf(s[c * 32 + 2 * t + 1], sl2, -m_use));
          sum += p0 + p1;
          pk[t] = pack_bf16x2(p0, p1);
        }
        tmem_st16(s_addr + c * 16, pk);
      }
      l_run += sum;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok) ok = warp_wait(o_full, static_cast<uint32_t>(n_tiles - 1) & 1u, ctx, kWhereO);
    tc_fence_after();

    // ---- sink epilogue (page "cf-1.com/news/6055759", fix 2) ----
    // new = max(row max, sink*log2e); r = 2^(old-new);
    // denominator' = denominator*r + 2^(sink*log2e - new); O = O_acc * r / denominator'.
    const float sink2 = p.sinks[h] * kLog2e;
    const float new_m = fmaxf(m_run, sink2);
    const float rs = (m_run == -INFINITY) ? 0.f : ex2_approx(m_run - new_m);
    const float l2 = l_run * rs + ((sink2 == -INFINITY) ? 0.f : ex2_approx(sink2 - new_m));
    const float oscale = (l2 > 0.f) ? rs / l2 : 0.f;
    const float lse_val = (l2 > 0.f) ? (new_m + log2f(l2)) * kLn2 : -INFINITY;

    if (ok) {
      // O (fp32, TMEM) -> bf16 -> swizzled staging tile in the Q buffer ->
      // TMA store; rows past the end of the sequence are clipped by the unit.
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(lane_base + C::kOCol + c * 32, o);
        tmem_wait_ld();
        uint8_t *chunk = sQ + (c >> 1) * (kBM * 128) + r * 128;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(o[8 * u + 0]) * oscale, __uint_as_float(o[8 * u + 1]) * oscale);
          v.y = pack_bf16x2(__uint_as_float(o[8 * u + 2]) * oscale, __uint_as_float(o[8 * u + 3]) * oscale);
          v.z = pack_bf16x2(__uint_as_float(o[8 * u + 4]) * oscale, __uint_as_float(o[8 * u + 5]) * oscale);
          v.w = pack_bf16x2(__uint_as_float(o[8 * u + 6]) * oscale, __uint_as_float(o[8 * u + 7]) * oscale);
          const int unit = (c & 1) * 4 + u;          // 16-byte unit within the 128-byte row
          *reinterpret_cast<uint4 *>(chunk + ((unit ^ (r & 7)) << 4)) = v;
        }
      }
      fence_proxy_async_smem();
    }
    named_barrier_sync(kBarEpilogue, kSoftmaxWarps * 32);
    if (threadIdx.x == 0 && !*abort_flag) {
      for (int c = 0; c < C::kChunks; ++c) tma_store_4d(&tmO, sQ + c * kBM * 128, c * 64, h, m0, b);
      tma_store_commit();
      tma_store_wait_all();
    }
    if (ok && p.lse != nullptr && i < p.L)
      p.lse[static_cast<int64_t>(b) * p.lse_sb + static_cast<int64_t>(h) * p.lse_sh + i] = lse_val;
  }

  // ---- teardown: all TMEM users are done before the allocator frees it ----
  if (is_tmem_warp(warp)) {
    tc_fence_before();
    named_barrier_sync(kBarTmem, kTmemThreads);
    if (warp == kMmaWarp) {
      tc_fence_after();
      tmem_dealloc(tmem, kTmemCols);
    }
  }
}

template <int D, int BN>
cudaError_t launch(const FwdArgs &a, cudaStream_t stream) {
  using C = Cfg<D, BN>;
  alignas(64) CUtensorMap mq, mk, mv, mo;
  cudaError_t e;
  if ((e = make_tma_bshd(&mq, a.q, a.B, a.L, a.Hq, D, a.q_s, kBM)) != cudaSuccess) return e;
  if ((e = make_tma_bshd(&mk, a.k, a.B, a.L, a.Hkv, D, a.k_s, BN)) != cudaSuccess) return e;
  if ((e = make_tma_bshd(&mv, a.v, a.B, a.L, a.Hkv, D, a.v_s, BN)) != cudaSuccess) return e;
  if ((e = make_tma_bshd(&mo, a.out, a.B, a.L, a.Hq, D, a.o_s, kBM)) != cudaSuccess) return e;
  Params p;
  p.L = a.L;
  p.Hq = a.Hq;
  p.W = a.W;
  p.group = a.Hq / a.Hkv;
  p.num_m_tiles = (a.L + kBM - 1) / kBM;
  p.scale_log2 = static_cast<float>(static_cast<double>(a.scale) * 1.4426950408889634);
  p.sinks = a.sinks;
  p.lse = a.lse;
  p.lse_sb = a.lse_s[0];
  p.lse_sh = a.lse_s[1];
  p.status = a.status;
  auto kern = fwd_tc_kernel<D, BN>;
  if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                C::kSmemBytes)) != cudaSuccess)
    return e;
  dim3 grid(p.num_m_tiles, a.Hq, a.B);
  kern<<<grid, kThreads, C::kSmemBytes, stream>>>(mq, mk, mv, mo, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_tc(const FwdArgs &a, cudaStream_t stream) {
  switch (a.D) {
    case 64: return launch<64, 128>(a, stream);
    case 128: return launch<128, 128>(a, stream);
    case 256: return launch<256, 64>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace attnsink
