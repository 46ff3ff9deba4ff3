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
// page describes (load / MMA / softmax roles, S and O accumulated in TMEM,
// two query tiles per CTA in ping-pong) as prior art; everything here is
// written for sm_100a directly.
//
// One CTA computes one 128-row query tile of one query head: 64-key tiles,
// two S buffers (S_{j+1} is computed while tile j is exponentiated), 256 TMEM
// columns at D <= 128, so two CTAs share each SM and their MMA streams and
// exponentials interleave (one CTA per SM at D = 256).  (Two heads of a kv
// group per CTA, sharing each K/V tile, measured as fast at W = 513 and
// slower at full causal with 64-key tiles and one MMA issuer per head, and
// slower everywhere with 128-key tiles.)  Warps (the head slot w is 0; the
// indexing is written per head):
//   0 .. 3       softmax / correction / epilogue, one thread per query row
//                (TMEM lane)
//   4            TMA producer: Q once per unit, then K_0, K_1, then V_j,
//                K_{j+2} per tile into a ring of shared-memory stages
//   5            TMEM allocator and MMA issuer: per key tile j, PV_j then the
//                S it frees a buffer for, so that the tensor cores compute
//                one tile while the softmax works on another.
// TMEM (columns): S buffer b at b*BN (P written as bf16 over its first BN/2
// columns), O after both S buffers.
// Only the K tiles that meet the window [m0-W+1, m0+127] are visited; the
// mask is applied on the tiles that cross the causal diagonal, the window's
// lower edge or the end of the sequence.
#include <math.h>

#include "kernels.h"
#include "ptx.cuh"

namespace attnsink {
namespace {

constexpr int kBM = 128;             // query rows per tile (= TMEM lanes)
constexpr uint32_t kBarTmem = 1;     // named barrier ids (0 = __syncthreads);
constexpr uint32_t kBarEpilogue0 = 2;  // 2 + w: epilogue of warpgroup w
constexpr uint32_t kBarVote0 = 4;      // 4 + w: warpgroup w's vote on going on
// Lazy rescaling: the running maximum (log2 units) only moves when a tile's
// maximum exceeds it by more than this; until then exponents stay <= 2^8.
constexpr float kRescaleThreshold = 8.0f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// Instruction mix of the exponentiation pass (chosen by measurement).
constexpr bool kPackedFma = true;   // f32x2 FMA for S*scale*log2e - m
constexpr bool kPackedAdd = true;   // f32x2 adds for the row sum
constexpr bool kFusedMax = true;    // tile maximum in the same pass (else: sum test)

// wait-location codes reported with ATTN_ETIMEOUT
enum : int { kWhereQ = 101, kWhereFull = 102, kWhereEmpty = 103, kWhereS = 104, kWhereP = 105,
             kWhereO = 106, kWhereAlign = 107 };

template <int D, int BN, int NH>
struct Cfg {
  static constexpr int kSoftmaxWarps = 4 * NH;
  static constexpr int kProducerWarp = 4 * NH;
  static constexpr int kMmaWarp = 4 * NH + 1;     // issuer of head w: kMmaWarp + w
  static constexpr int kWarps = 4 * NH + 2;
  static constexpr int kThreads = kWarps * 32;
  // (The head-slot indexing below is written for NH heads per CTA; one is
  // built.  Two heads per CTA, with 64- and 128-key tiles, were measured with
  // earlier versions of this kernel and were slower or no faster.)
  static_assert(NH == 1, "one query head per CTA");
  // The warps that touch TMEM: the softmax warpgroups and the MMA warp.  This
  // is the single definition of the TMEM allocation barrier's participant
  // set; the barrier count and the participation test both derive from it.
  static constexpr uint32_t kTmemWarpMask = ((1u << (4 * NH)) - 1u) | (((1u << NH) - 1u) << kMmaWarp);
  static_assert(kMmaWarp + NH <= kWarps, "issuer warps");
  static constexpr uint32_t kTmemThreads = 32u * __builtin_popcount(kTmemWarpMask);

  static constexpr int kChunks = D / 64;          // 64-channel (128-byte) column chunks
  static constexpr int kBarBytes = 256;           // mbarriers, TMEM base, abort flag
  static constexpr int kQTileBytes = kBM * D * 2;
  static constexpr int kQBufBytes = NH * kQTileBytes;   // one unit's Q tiles (later its O staging)
  static constexpr int kQBytes = 2 * kQBufBytes;        // double buffered across units
  static constexpr int kTileBytes = BN * D * 2;   // one K or V tile
  // two S buffers: S_{j+1} is computed while S_j is exponentiated
  static constexpr int kSBuf = 2;
  static constexpr int kColsUsed = NH * (kSBuf * BN + D);
  static constexpr uint32_t kTmemCols = kColsUsed <= 256 ? 256u : 512u;
  static constexpr int kCtasPerSm = (kTmemCols == 256u) ? 2 : 1;
  // per-CTA shared-memory budget: the SM's 228 KB shared by kCtasPerSm CTAs,
  // each also reserving 1 KB, minus the barrier block (the dynamic shared
  // memory is declared 1024-byte aligned, so no alignment slack: at D = 128
  // with two CTAs per SM that is what leaves room for a third ring stage)
  static constexpr int kBudget = (228 * 1024) / kCtasPerSm - 1024 - kBarBytes;
  static constexpr int kStagesRaw = (kBudget - kQBytes) / kTileBytes;
  static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
  static constexpr int kRingBytes = kStages * kTileBytes;
  static constexpr int kBarOffset = kQBytes + kRingBytes;
  static constexpr int kSmemBytes = kBarOffset + kBarBytes;
  static constexpr uint32_t kSCol(int w, int buf) { return static_cast<uint32_t>((kSBuf * w + buf) * BN); }
  static constexpr uint32_t kOCol(int w) { return static_cast<uint32_t>(kSBuf * NH * BN + w * D); }
  static_assert(kStages >= 2, "need at least two ring stages");
  // full/empty per stage, q_full/q_empty [2], s_full/p_full [NH][2],
  // pv_done/o_full/o_drained [NH], mma_done; then the TMEM base and the abort flag
  static_assert((2 * kStages + 4 + 7 * NH + 1) * 8 + 8 <= kBarBytes, "barrier block");
  static_assert(kColsUsed <= 512, "TMEM budget");
  static_assert(kSmemBytes <= 227 * 1024, "shared-memory budget");
};

template <int D, int BN, int NH>
__host__ __device__ constexpr bool is_tmem_warp(int w) {
  return (Cfg<D, BN, NH>::kTmemWarpMask >> w) & 1u;
}

struct Params {
  int L, Hq, W, group, num_m_tiles, B, num_units;
  float scale_log2;
  const float *sinks;
  float *lse;
  int64_t lse_sb, lse_sh;
  int *status;
  // Packed variable-length sequences (null: a [B, L] batch).  Sequence b is
  // rows cu_seqlens[b] .. cu_seqlens[b+1]-1 of [T, H, D] tensors; the last,
  // ragged query tile of a sequence is stored row by row through `out`.
  const int *cu_seqlens;
  int T;
  __nv_bfloat16 *out;
  int64_t o_sr, o_sh;
  float *max_logit;                        // [B, Hq] (stride ml_sb), kMaxLogit only
  int64_t ml_sb;
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

// Columns outside [lo, hi] of a 32-column chunk starting at column c0 -> -inf.
__device__ __forceinline__ void mask_chunk(uint32_t (&x)[32], int c0, int lo, int hi) {
#pragma unroll
  for (int t = 0; t < 32; ++t)
    if (c0 + t < lo || c0 + t > hi) x[t] = __float_as_uint(-INFINITY);
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ uint64_t f2pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}

__device__ __forceinline__ void f2unpack(uint64_t r, float &a, float &b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}

__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// P = 2^(S*scale*log2e - m_use) for one row tile held in registers (sv),
// written as bf16 over the first BN/2 columns at p_addr; returns the fp32 sum
// of P, and with kMax also the tile's raw maximum in tmax.
template <int BN, bool kMax>
__device__ __forceinline__ float exp_tile(const uint32_t (&sv)[BN / 32][32], uint32_t p_addr,
                                          float sl2, float m_use, uint32_t cls_none, float &tmax) {
  const uint64_t sl2x2 = f2pack(sl2, sl2);
  const uint64_t negm2 = f2pack(-m_use, -m_use);
  uint64_t acc2[2] = {f2pack(0.f, 0.f), f2pack(0.f, 0.f)};
  float accs[4] = {0.f, 0.f, 0.f, 0.f};
  float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int c = 0; c < BN / 32; ++c) {
    uint32_t pk[16];
    if (cls_none >> c & 1u) {
#pragma unroll
      for (int t = 0; t < 16; ++t) pk[t] = 0u;
    } else {
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        const float s0 = __uint_as_float(sv[c][2 * t]), s1 = __uint_as_float(sv[c][2 * t + 1]);
        if (kMax) mx[t & 3] = fmax3(mx[t & 3], s0, s1);
        float z0, z1;
        if (kPackedFma) {
          f2unpack(fma2(f2pack(s0, s1), sl2x2, negm2), z0, z1);
        } else {
          z0 = fmaf(s0, sl2, -m_use);
          z1 = fmaf(s1, sl2, -m_use);
        }
        const float p0 = ex2_approx(z0), p1 = ex2_approx(z1);
        if (kPackedAdd) {
          acc2[t & 1] = add2(acc2[t & 1], f2pack(p0, p1));
        } else {
          accs[t & 3] += p0;
          accs[(t + 2) & 3] += p1;
        }
        pk[t] = pack_bf16x2(p0, p1);
      }
    }
    tmem_st16(p_addr + c * 16, pk);
  }
  if (kMax) tmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
  if (kPackedAdd) {
    float a0, a1, b0, b1;
    f2unpack(acc2[0], a0, a1);
    f2unpack(acc2[1], b0, b1);
    return (a0 + a1) + (b0 + b1);
  }
  return (accs[0] + accs[1]) + (accs[2] + accs[3]);
}

// Raw maximum of the non-empty chunks of a row tile held in registers.
template <int BN>
__device__ __forceinline__ float tile_max(const uint32_t (&sv)[BN / 32][32], uint32_t cls_none) {
  float a[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) a[u] = -INFINITY;
#pragma unroll
  for (int c = 0; c < BN / 32; ++c) {
    if (cls_none >> c & 1u) continue;
#pragma unroll
    for (int t = 0; t < 16; ++t)
      a[t & 7] = fmax3(a[t & 7], __uint_as_float(sv[c][2 * t]), __uint_as_float(sv[c][2 * t + 1]));
  }
  return fmax3(fmax3(a[0], a[1], a[2]), fmax3(a[3], a[4], a[5]), fmaxf(a[6], a[7]));
}

// One key tile of the online softmax for the calling thread's row (its TMEM
// lane): read S (one TMEM round trip), mask, update the running state and
// write P over S.  From the second tile on, P is computed against the running
// maximum while the tile maximum is found in the same pass; only if a row's
// maximum then grew by more than the lazy-rescale threshold (rare after the
// first tiles) does its warp rescale O and recompute P.  Returns false if a
// bounded wait ran out.
template <int D, int BN>
__device__ __forceinline__ bool softmax_tile(uint32_t lane_base, uint32_t s_col, uint32_t o_col,
                                             int j, int g, float sl2, int lo, int hi, uint32_t cls_mask,
                                             uint32_t cls_none, float &m_run, float &l_run,
                                             float &row_max,
                                             uint64_t *pv_done,
                                             const WaitCtx &ctx) {
  constexpr int NC = BN / 32;
  uint32_t sv[NC][32];
#pragma unroll
  for (int c = 0; c < NC; ++c)
    if (!(cls_none >> c & 1u)) tmem_ld32(lane_base + s_col + c * 32, sv[c]);
  tmem_wait_ld();
#pragma unroll
  for (int c = 0; c < NC; ++c)
    if (cls_mask >> c & 1u) mask_chunk(sv[c], c * 32, lo, hi);
  float tm;
  if (j == 0) {
    // first tile: nothing accumulated yet, so take the maximum first
    const float mt2 = tile_max<BN>(sv, cls_none) * sl2;
    row_max = fmaxf(row_max, mt2);
    if (mt2 > m_run + kRescaleThreshold) m_run = mt2;
    l_run = exp_tile<BN, false>(sv, lane_base + s_col, sl2, (m_run == -INFINITY) ? 0.f : m_run,
                                cls_none, tm);
    return true;
  }
  const float sum = exp_tile<BN, kFusedMax>(sv, lane_base + s_col, sl2,
                                            (m_run == -INFINITY) ? 0.f : m_run, cls_none, tm);
  // Without the fused maximum: every P <= 2^threshold when the tile's sum is
  // at most that, so no row can have moved past the threshold; otherwise the
  // maximum is taken now (and usually turns out not to have moved either).
  if (!kFusedMax) tm = (sum <= 256.f) ? -INFINITY : tile_max<BN>(sv, cls_none);
  const float mt2 = tm * sl2;
  row_max = fmaxf(row_max, mt2);
  const bool grow = mt2 > m_run + kRescaleThreshold;
  if (!__any_sync(0xffffffffu, grow)) {
    l_run += sum;
    return true;
  }
  // Rare path: some row's maximum moved.  O holds sum_{t<j} P_t V_t once
  // PV_{j-1} has finished (S_j finished implies that the PVs issued before it,
  // up to PV_{j-kSBuf}, finished, so the barrier is at most one phase behind
  // and the parity wait is exact); rescale it and recompute P.
  float alpha = 1.f;
  if (grow) {
    alpha = ex2_approx(m_run - mt2);               // 0 while nothing was seen yet
    m_run = mt2;
  }
  if (!warp_wait(pv_done, static_cast<uint32_t>(g - 1) & 1u, ctx, kWhereO)) return false;
  tc_fence_after();
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    uint32_t o[32];
    tmem_ld32(lane_base + o_col + c * 32, o);
    tmem_wait_ld();
#pragma unroll
    for (int t = 0; t < 32; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * alpha);
    tmem_st32(lane_base + o_col + c * 32, o);
  }
  tmem_wait_st();
  l_run = l_run * alpha + exp_tile<BN, false>(sv, lane_base + s_col, sl2,
                                              (m_run == -INFINITY) ? 0.f : m_run, cls_none, tm);
  return true;
}

// kPacked: packed variable-length sequences (Params::cu_seqlens); a separate
// instantiation, so that the batched kernel carries none of its code.
__global__ void max_logit_init_kernel(float *ml, int64_t sb, int B, int Hq) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t < B * Hq) ml[static_cast<int64_t>(t / Hq) * sb + t % Hq] = -INFINITY;
}

// Float maximum by integer atomics: non-negative floats order as signed ints,
// negative ones in reverse as unsigned ints (so -inf, the start value, loses
// to every other value).
__device__ __forceinline__ void atomic_max_float(float *addr, float v) {
  if (v >= 0.f)
    atomicMax(reinterpret_cast<int *>(addr), __float_as_int(v));
  else
    atomicMin(reinterpret_cast<unsigned int *>(addr), __float_as_uint(v));
}

// kMaxLogit: also the largest content logit scale*<q_i,k_j> over every row and
// visible key of each (sequence, head), into Params::max_logit (atomic max).
template <int D, int BN, int NH, bool kPacked, bool kMaxLogit>
__global__ void __launch_bounds__(Cfg<D, BN, NH>::kThreads, Cfg<D, BN, NH>::kCtasPerSm)
    fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                  const Params p) {
  using C = Cfg<D, BN, NH>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // (128-byte swizzled tiles need 1024-byte aligned addresses; the budget
  // has no slack for aligning by hand, so a base off the declared alignment
  // is reported and nothing runs)
  if (reinterpret_cast<uintptr_t>(smem_raw) & 1023u) {
    if (threadIdx.x == 0) report_launch_error(p.status, kWhereAlign);
    return;
  }
  uint8_t *smem = smem_raw;
  uint8_t *sQ = smem;                       // [2] units' Q tiles, later their O staging
  uint8_t *sRing = smem + C::kQBytes;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarOffset);
  uint64_t *empty = full + C::kStages;
  uint64_t *q_full = empty + C::kStages;    // [2] a unit's Q landed in buffer u%2
  uint64_t *q_empty = q_full + 2;           // [2] buffer u%2's O store has read it (NH arrivals)
  uint64_t *s_full = q_empty + 2;           // [NH][2] S^w ready in S buffer
  uint64_t *p_full = s_full + 2 * NH;       // [NH][2] P^w ready in S buffer (O^w rescaled)
  uint64_t *pv_done = p_full + 2 * NH;      // [NH] one PV^w finished
  uint64_t *o_full = pv_done + NH;          // [NH] a unit's last PV^w finished
  uint64_t *o_drained = o_full + NH;        // [NH] O^w of a unit read out of TMEM
  uint64_t *mma_done = o_drained + NH;      // every MMA of the CTA finished
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
  int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
  const WaitCtx ctx{abort_flag, p.status, wait_limit_ns(p.status)};

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int HP = p.Hq / NH;                 // head groups (units per position and batch)
  // Work units: (query tile, head group, batch), latest query tiles first (they
  // see the most keys under a causal window), head groups fastest so that the
  // CTAs running at the same time share K/V tiles in L2.  CTA c takes units
  // c, c + gridDim.x, ...
  // A unit's sequence has `len` positions starting at row `row0` of the
  // row dimension, in batch slice bc() of the tensor maps; with packed
  // sequences a unit past its sequence's end is empty (n_tiles = 0) and every
  // role skips it.
  struct Unit {
    int m0, h0, b, kt0, n_tiles, len, row0;
  };
  constexpr bool packed = kPacked;
  auto bc = [&](const Unit &t) { return packed ? 0 : t.b; };
  auto unit_at = [&](int u) {
    Unit t;
    const int per_m = HP * p.B;
    const int mt = p.num_m_tiles - 1 - u / per_m;
    const int r = u - (u / per_m) * per_m;
    t.h0 = (r % HP) * NH;
    t.b = r / HP;
    t.m0 = mt * kBM;
    if constexpr (packed) {
      // offsets clamped to [0, T], so that a malformed table never moves a
      // store outside the tensors
      t.row0 = min(max(p.cu_seqlens[t.b], 0), p.T);
      t.len = min(max(p.cu_seqlens[t.b + 1], t.row0), p.T) - t.row0;
    } else {
      t.row0 = 0;
      t.len = p.L;
    }
    const int row_last = min(t.len - 1, t.m0 + kBM - 1);
    t.kt0 = max(0, t.m0 - p.W + 1) / BN;
    t.n_tiles = t.m0 < t.len ? row_last / BN - t.kt0 + 1 : 0;
    return t;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NH);              // each head's issuer frees the stage
    }
    for (int qb = 0; qb < 2; ++qb) {
      mbar_init(&q_full[qb], 1);
      mbar_init(&q_empty[qb], NH);
    }
    for (int w = 0; w < NH; ++w) {
      for (int buf = 0; buf < 2; ++buf) {
        mbar_init(&s_full[2 * w + buf], 1);
        mbar_init(&p_full[2 * w + buf], 128);
      }
      mbar_init(&pv_done[w], 1);
      mbar_init(&o_full[w], 1);
      mbar_init(&o_drained[w], 128);
    }
    mbar_init(mma_done, NH);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // ---- TMEM allocation (page "cf-1.com/news/6055759", fix 1) ----
  // The MMA warp allocates; every TMEM warp then meets at one named barrier
  // whose count is exactly the number of threads in kTmemWarpMask, and only
  // after it reads the column base.
  if (warp == C::kMmaWarp) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  uint32_t tmem = 0;
  if (is_tmem_warp<D, BN, NH>(warp)) {
    tc_fence_before();
    named_barrier_sync(kBarTmem, C::kTmemThreads);
    tc_fence_after();
    tmem = *tmem_slot;
  }

  if (warp >= C::kSoftmaxWarps) {
  if (warp == C::kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int slot = 0, q_loaded = 0;
      bool ok = true;
      auto load = [&](const CUtensorMap *map, int kt, int b) {
        const int s = slot % C::kStages;
        const uint32_t use = static_cast<uint32_t>(slot / C::kStages);
        if (slot >= C::kStages && !mbar_wait(&empty[s], (use & 1u) ^ 1u, ctx, kWhereEmpty)) {
          ok = false;
          return;
        }
        mbar_arrive_expect_tx(&full[s], C::kTileBytes);
        uint8_t *dst = sRing + s * C::kTileBytes;
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_4d(dst + c * BN * 128, map, &full[s], c * 64, 0, kt * BN, b);
        ++slot;
      };
      int ul = -1;                            // units that are not empty, so far
      for (int u = blockIdx.x; ok && u < p.num_units; u += gridDim.x) {
        const Unit t = unit_at(u);
        if (packed && t.n_tiles <= 0) continue;
        ++ul;
        const int qb = ul & 1;
        // the buffer's previous unit has stored its O out of it
        if (ul >= 2 &&
            !mbar_wait(&q_empty[qb], static_cast<uint32_t>((ul >> 1) - 1) & 1u, ctx, kWhereQ)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&q_full[qb], C::kQBufBytes);
        for (int w = 0; w < NH; ++w)
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_4d(sQ + qb * C::kQBufBytes + w * C::kQTileBytes + c * kBM * 128, &tmQ,
                        &q_full[qb], c * 64, t.h0 + w, t.row0 + t.m0, bc(t));
        q_loaded = ul + 1;
        const int hk = t.h0 / p.group;
        // the order the MMA warp consumes: K_0 .. K_{kSBuf-1}, then per tile
        // j: V_j, K_{j+kSBuf}
        auto kv = [&](const CUtensorMap *map, int kt) {
          const int s = slot % C::kStages;
          const uint32_t use = static_cast<uint32_t>(slot / C::kStages);
          if (slot >= C::kStages && !mbar_wait(&empty[s], (use & 1u) ^ 1u, ctx, kWhereEmpty)) {
            ok = false;
            return;
          }
          mbar_arrive_expect_tx(&full[s], C::kTileBytes);
          uint8_t *dst = sRing + s * C::kTileBytes;
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_4d(dst + c * BN * 128, map, &full[s], c * 64, hk, t.row0 + kt * BN, bc(t));
          ++slot;
        };
        for (int jj = 0; ok && jj < C::kSBuf && jj < t.n_tiles; ++jj) kv(&tmK, t.kt0 + jj);
        for (int j = 0; ok && j < t.n_tiles; ++j) {
          kv(&tmV, t.kt0 + j);
          if (ok && j + C::kSBuf < t.n_tiles) kv(&tmK, t.kt0 + j + C::kSBuf);
        }
      }
      (void)load;
      // Before this warp leaves, the copies it issued have landed: the CTA (and
      // its shared memory) must outlive them even when the other roles gave
      // up early.  Only the last two Q loads and the last kStages K/V tiles
      // can still be in flight (every earlier one was waited for before its
      // buffer was reused).  In a normal run they are long done.
      for (int uq = max(0, q_loaded - 2); uq < q_loaded; ++uq)
        drain_wait(&q_full[uq & 1], static_cast<uint32_t>(uq >> 1) & 1u);
      for (int t = max(0, slot - C::kStages); t < slot; ++t)
        drain_wait(&full[t % C::kStages], static_cast<uint32_t>(t / C::kStages) & 1u);
    }
    __syncwarp();
  } else if (warp >= C::kMmaWarp && warp < C::kMmaWarp + NH) {
    // ----------------------------------------------------------------- MMA
    const int w = warp - C::kMmaWarp;        // this warp issues head w's products
    if (lane == 0) {
      constexpr uint32_t idesc_qk = umma_idesc_bf16(kBM, BN, 0, 0);  // Q, K both K-major
      constexpr uint32_t idesc_pv = umma_idesc_bf16(kBM, D, 0, 1);   // V is N-major
      // descriptor words: 128-byte swizzle, 8-row groups 1024 bytes apart;
      // K-major operands (Q, K) need no leading offset, the N-major V tile has
      // its 64-channel chunks BN*128 bytes apart
      const uint32_t desc_hi = umma_desc_hi_sw128(1024);
      const uint32_t q_lo = umma_desc_lo(smem_u32(sQ), 16);
      const uint32_t ring_lo_k = umma_desc_lo(smem_u32(sRing), 16);
      const uint32_t ring_lo_v = umma_desc_lo(smem_u32(sRing), BN * 128);
      bool ok = true;
      int slot = 0;
      auto acquire = [&](int &s) {
        s = slot % C::kStages;
        ok = ok && mbar_wait(&full[s], static_cast<uint32_t>(slot / C::kStages) & 1u, ctx,
                             kWhereFull);
        ++slot;
        tc_fence_after();
        return ok;
      };
      // S^w_g = Q^w K^T into S buffer g%kSBuf of head w, Q from buffer qbuf
      // (overwriting the P^w that the PV^w issued before it has consumed: the
      // tensor pipe runs in order)
      auto issue_s = [&](int w, int ks, int g, int qbuf) {
        const uint32_t a0 = q_lo + ((qbuf * C::kQBufBytes + w * C::kQTileBytes) >> 4);
        const uint32_t b0 = ring_lo_k + ks * (C::kTileBytes >> 4);
        const uint32_t d = tmem + C::kSCol(w, g % C::kSBuf);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          // 16 channels = 32 bytes along the swizzled row; 64-channel chunks apart
          umma_ss_w(d, a0 + (kk >> 2) * (kBM * 128 >> 4) + (kk & 3) * 2, desc_hi,
                    b0 + (kk >> 2) * (BN * 128 >> 4) + (kk & 3) * 2, desc_hi, idesc_qk,
                    kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[2 * w + g % C::kSBuf]);
      };
      // O^w += P^w_g V with P^w_g (bf16 pairs) in the first BN/2 columns of
      // its S buffer; j = 0 starts a unit's O^w
      auto issue_pv = [&](int w, int vs, int g, int j) {
        const uint32_t b0 = ring_lo_v + vs * (C::kTileBytes >> 4);
        const uint32_t a0 = tmem + C::kSCol(w, g % C::kSBuf);
        const uint32_t d = tmem + C::kOCol(w);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          umma_ts_w(d, a0 + kk * 8, b0 + kk * (16 * 128 >> 4), desc_hi, idesc_pv,
                    (j > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&pv_done[w]);
      };
      int jg = 0;                            // tiles of earlier units (barrier phases)
      for (int ul = 0, u = blockIdx.x; ok && u < p.num_units; u += gridDim.x) {
        const Unit t = unit_at(u);
        if (packed && t.n_tiles <= 0) continue;   // ul counts the units that are not empty
        const int qb = ul & 1;
        int ks = 0, vs = 0;
        {
          if (!mbar_wait(&q_full[qb], static_cast<uint32_t>(ul >> 1) & 1u, ctx, kWhereQ)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int jj = 0; ok && jj < C::kSBuf && jj < t.n_tiles; ++jj) {
            if (!acquire(ks)) break;
            issue_s(w, ks, jg + jj, qb);
            umma_commit(&empty[ks]);
          }
        }
        for (int j = 0; ok && j < t.n_tiles; ++j) {
          const int g = jg + j;
          const bool more = j + C::kSBuf < t.n_tiles;
          const bool last = j == t.n_tiles - 1;
          if (!acquire(vs)) break;
          {
            if (!mbar_wait(&p_full[2 * w + g % C::kSBuf], static_cast<uint32_t>(g / C::kSBuf) & 1u,
                           ctx, kWhereP)) {
              ok = false;
              break;
            }
            // the first PV of a unit overwrites O^w: the previous unit's O^w
            // must have been read out of TMEM
            if (j == 0 && ul > 0 &&
                !mbar_wait(&o_drained[w], static_cast<uint32_t>(ul - 1) & 1u, ctx, kWhereO)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_pv(w, vs, g, j);
            if (last) umma_commit(&o_full[w]);   // this unit's O^w is complete
            umma_commit(&empty[vs]);
            // the S that this PV frees the buffer for: S_{j+kSBuf}
            if (more) {
              if (!acquire(ks)) break;
              issue_s(w, ks, g + C::kSBuf, qb);
              umma_commit(&empty[ks]);
            }
          }
        }
        jg += t.n_tiles;
        ++ul;
      }
      // Every tensor-core operation of this CTA has finished before teardown.
      umma_commit(mma_done);
      drain_wait(mma_done, 0);
    }
    __syncwarp();
    // ---- teardown: all TMEM users are done before the allocator frees it ----
    tc_fence_before();
    named_barrier_sync(kBarTmem, C::kTmemThreads);
    tc_fence_after();
    if (warp == C::kMmaWarp) tmem_dealloc(tmem, C::kTmemCols);
  }
  } else {
    // ------------------------------------------- softmax / correction / epilogue
    const int w = warp >> 2;                         // head slot of this warpgroup
    const int r = threadIdx.x & 127;                 // tile row == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t o_col = C::kOCol(w);
    const float sl2 = p.scale_log2;
    bool ok = true;
    int jg = 0;
    int pending_qb = -1;                             // buffer whose O store may still read it
    int ul = -1;                                     // units that are not empty, so far
    for (int u = blockIdx.x; ok && u < p.num_units; u += gridDim.x) {
      const Unit t = unit_at(u);
      if (packed && t.n_tiles <= 0) continue;
      ++ul;
      const int qb = ul & 1;
      const int h = t.h0 + w;
      const int i = t.m0 + r;                        // query position
      float m_run = -INFINITY;                       // running max, log2 units
      float row_max = -INFINITY;                     // exact row maximum, log2 units
      float l_run = 0.f;                             // running denominator
      for (int j = 0; ok && j < t.n_tiles; ++j) {
        const int g = jg + j;
        const uint32_t s_col = C::kSCol(w, g % C::kSBuf);
        if (!warp_wait(&s_full[2 * w + g % C::kSBuf], static_cast<uint32_t>(g / C::kSBuf) & 1u,
                       ctx, kWhereS)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int kbase = (t.kt0 + j) * BN;
        // Tile-uniform test: does any (row, key) of this tile fall outside the
        // causal window or past the end of the sequence?
        const bool edge = (kbase + BN - 1 > t.m0) || (kbase < t.m0 + kBM - p.W) || (kbase + BN > t.len);
        const int lo = i - p.W + 1 - kbase;          // first visible column
        const int hi = min(i, t.len - 1) - kbase;    // last visible column
        // Per 32-column chunk, a warp-uniform class: every lane's visible
        // interval [lo, hi] covers the chunk (no mask), misses it (no work:
        // P = 0), or cuts it (per-element mask).
        uint32_t cls_mask = 0, cls_none = 0;         // bit c: chunk c mixed / empty
        if (edge) {
#pragma unroll
          for (int c = 0; c < BN / 32; ++c) {
            const bool all_in = __all_sync(0xffffffffu, lo <= c * 32 && hi >= c * 32 + 31);
            const bool all_out = __all_sync(0xffffffffu, hi < c * 32 || lo > c * 32 + 31);
            cls_none |= (all_out ? 1u : 0u) << c;
            cls_mask |= (!all_in && !all_out ? 1u : 0u) << c;
          }
        }
        if (!softmax_tile<D, BN>(lane_base, s_col, o_col, j, g, sl2, lo, hi, cls_mask, cls_none,
                                 m_run, l_run, row_max, &pv_done[w], ctx)) {
          ok = false;
          break;
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[2 * w + g % C::kSBuf]);
        if (j == 0 && pending_qb >= 0 && r == 0) {
          // The previous unit's O store has long finished reading its staging
          // tile: hand the buffer back for the Q of a later unit.
          tma_store_wait_read();
          mbar_arrive(&q_empty[pending_qb]);
          pending_qb = -1;
        }
      }
      jg += t.n_tiles;
      bool w_ok = false;
      if (ok) w_ok = warp_wait(&o_full[w], static_cast<uint32_t>(ul) & 1u, ctx, kWhereO);
      // Every warp of the warpgroup reaches this vote once per unit (a warp
      // whose bounded wait ran out leaves its tile loop early and comes here),
      // so the epilogue's barrier below is met by all four warps or by none.
      ok = named_barrier_and(kBarVote0 + w, 128, w_ok);
      if (!ok) break;
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

      // O^w (fp32, TMEM) -> bf16 -> swizzled staging tile (this unit's Q^w
      // buffer, no longer read) -> TMA store; rows past the end of a batch
      // tensor are clipped by the store.  The ragged last tile of a packed
      // sequence is instead written row by row from registers (rows past the
      // sequence's end belong to the next sequence).  Once O^w is out of TMEM
      // the next unit's PV^w may overwrite it.
      uint8_t *stage = sQ + qb * C::kQBufBytes + w * C::kQTileBytes;
      const bool direct = packed && t.m0 + kBM > t.len;
      // the next 32-column chunk is read while this one is converted
      auto convert = [&](int c, const uint32_t (&o)[32]) {
        uint8_t *chunk = stage + (c >> 1) * (kBM * 128) + r * 128;
#pragma unroll
        for (int uu = 0; uu < 4; ++uu) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(o[8 * uu + 0]) * oscale, __uint_as_float(o[8 * uu + 1]) * oscale);
          v.y = pack_bf16x2(__uint_as_float(o[8 * uu + 2]) * oscale, __uint_as_float(o[8 * uu + 3]) * oscale);
          v.z = pack_bf16x2(__uint_as_float(o[8 * uu + 4]) * oscale, __uint_as_float(o[8 * uu + 5]) * oscale);
          v.w = pack_bf16x2(__uint_as_float(o[8 * uu + 6]) * oscale, __uint_as_float(o[8 * uu + 7]) * oscale);
          if (direct) {
            if (i < t.len)
              *reinterpret_cast<uint4 *>(p.out + static_cast<int64_t>(t.row0 + i) * p.o_sr +
                                         static_cast<int64_t>(h) * p.o_sh + c * 32 + uu * 8) = v;
          } else {
            const int unit = (c & 1) * 4 + uu;      // 16-byte unit within the 128-byte row
            *reinterpret_cast<uint4 *>(chunk + ((unit ^ (r & 7)) << 4)) = v;
          }
        }
      };
      static_assert(D % 64 == 0, "chunks are converted in pairs");
      // one chunk in flight (two measured 1.6 % slower: registers)
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(lane_base + o_col + c * 32, o);
        tmem_wait_ld_dep(o);
        convert(c, o);
      }
      tc_fence_before();
      mbar_arrive(&o_drained[w]);
      fence_proxy_async_smem();
      if (w == 0)
        named_barrier_sync(kBarEpilogue0, 128);
      else
        named_barrier_sync(kBarEpilogue0 + 1, 128);
      if (r == 0) {
        if (!direct) {
          for (int c = 0; c < C::kChunks; ++c)
            tma_store_4d(&tmO, stage + c * kBM * 128, c * 64, h, t.row0 + t.m0, bc(t));
          tma_store_commit();
        }
        pending_qb = qb;                           // released at the next unit's first tile
      }
      if (p.lse != nullptr && i < t.len)
        p.lse[(packed ? t.row0 : static_cast<int64_t>(t.b) * p.lse_sb) + static_cast<int64_t>(h) * p.lse_sh +
              i] = lse_val;
      if constexpr (kMaxLogit) {
        // the unit's largest logit (log2 units back to natural): warp
        // maximum, then one atomic per warp
        float v = (i < t.len) ? row_max * kLn2 : -INFINITY;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
        if ((r & 31) == 0 && v > -INFINITY) atomic_max_float(&p.max_logit[static_cast<int64_t>(t.b) * p.ml_sb + h], v);
      }
    }
    // stores must have read shared memory before the CTA leaves
    if (r == 0) tma_store_wait_all();
    // teardown: this warp's TMEM reads are complete before the allocator frees it
    tc_fence_before();
    named_barrier_sync(kBarTmem, C::kTmemThreads);
  }
}

template <int D, int BN, int NH, bool kPacked, bool kMaxLogit = false>
cudaError_t launch(const FwdArgs &a, cudaStream_t stream) {
  using C = Cfg<D, BN, NH>;
  alignas(64) CUtensorMap mq, mk, mv, mo;
  cudaError_t e;
  // packed sequences: one [T, H, D] slice; else the [B, L, H, D] batch
  const int64_t nb = a.cu_seqlens != nullptr ? 1 : a.B;
  const int64_t nrow = a.cu_seqlens != nullptr ? a.T : a.L;
  if ((e = make_tma_bshd(&mq, a.q, nb, nrow, a.Hq, D, a.q_s, kBM)) != cudaSuccess) return e;
  if ((e = make_tma_bshd(&mk, a.k, nb, nrow, a.Hkv, D, a.k_s, BN)) != cudaSuccess) return e;
  if ((e = make_tma_bshd(&mv, a.v, nb, nrow, a.Hkv, D, a.v_s, BN)) != cudaSuccess) return e;
  if ((e = make_tma_bshd(&mo, a.out, nb, nrow, a.Hq, D, a.o_s, kBM)) != cudaSuccess) return e;
  Params p;
  p.L = a.L;
  p.Hq = a.Hq;
  p.W = a.W;
  p.group = a.Hq / a.Hkv;
  p.num_m_tiles = (a.L + kBM - 1) / kBM;
  p.B = a.B;
  p.num_units = p.num_m_tiles * (a.Hq / NH) * a.B;
  p.scale_log2 = static_cast<float>(static_cast<double>(a.scale) * 1.4426950408889634);
  p.sinks = a.sinks;
  p.lse = a.lse;
  p.lse_sb = a.lse_s[0];
  p.lse_sh = a.lse_s[1];
  p.status = a.status;
  p.cu_seqlens = a.cu_seqlens;
  p.T = a.T;
  p.out = static_cast<__nv_bfloat16 *>(a.out);
  p.o_sr = a.o_s[1];
  p.o_sh = a.o_s[2];
  p.max_logit = a.max_logit;
  p.ml_sb = a.ml_sb;
  if (kMaxLogit) {
    // every entry starts at -inf; the kernel's units raise it
    if ((e = launch_max_logit_init(a.max_logit, a.ml_sb, a.B, a.Hq, stream)) != cudaSuccess) return e;
  }
  auto kern = fwd_tc_kernel<D, BN, NH, kPacked, kMaxLogit>;
  static bool attr_set[64] = {};  // once per device (per instantiation)
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  C::kSmemBytes)) != cudaSuccess)
      return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  static int sm_count[64] = {};
  if (dev >= 0 && dev < 64 && sm_count[dev] == 0)
    if ((e = cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return e;
  const int sms = (dev >= 0 && dev < 64) ? sm_count[dev] : 148;
  const int slots = sms * C::kCtasPerSm;
  dim3 grid(p.num_units < slots ? p.num_units : slots);
  kern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(mq, mk, mv, mo, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_max_logit_init(float *ml, int64_t sb, int B, int Hq, cudaStream_t stream) {
  const int n = B * Hq;
  if (n <= 0) return cudaSuccess;
  max_logit_init_kernel<<<(n + 255) / 256, 256, 0, stream>>>(ml, sb, B, Hq);
  return cudaGetLastError();
}

cudaError_t launch_fwd_tc(const FwdArgs &a, cudaStream_t stream) {
  // One query head per CTA, 64-key tiles with two S buffers, two CTAs per SM
  // (one at D = 256), for every group size.
  const bool packed = a.cu_seqlens != nullptr;
  const bool ml = a.max_logit != nullptr;   // (batched inputs only)
  if (packed && ml) return cudaErrorInvalidValue;
  switch (a.D) {
    case 64:
      if (packed) return launch<64, 64, 1, true>(a, stream);
      return ml ? launch<64, 64, 1, false, true>(a, stream) : launch<64, 64, 1, false>(a, stream);
    case 128:
      if (packed) return launch<128, 64, 1, true>(a, stream);
      return ml ? launch<128, 64, 1, false, true>(a, stream) : launch<128, 64, 1, false>(a, stream);
    case 256:
      if (packed) return launch<256, 64, 1, true>(a, stream);
      return ml ? launch<256, 64, 1, false, true>(a, stream) : launch<256, 64, 1, false>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace attnsink
