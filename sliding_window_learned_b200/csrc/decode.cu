// decode.cu -- single-token split-KV decode with a learned per-head sink.
//
// Three kernels on one stream, no host synchronisation:
//   plan     reads seqlens on the device; splits each sequence's visible key
//            range [max(0, n-W), n) into chunks of `chunk` keys and lays the
//            splits out contiguously (split_base[b] = exclusive prefix sum).
//            For a paged cache the range first starts at the 64-key boundary
//            below max(0, n-W), so that no key tile straddles two pages; the
//            keys before the window are masked.
//   split    persistent: one work item = (split, kv head).  A TMA producer
//            warp streams 64-key K/V tiles of that head into a ring of stages
//            (for a paged cache, each tile from the pool page(s) the block
//            table names: one box per tile, or for pages of 16 or 32
//            positions one box per page holding every channel chunk, through
//            a 5-D view of the pool);
//            the consumer warps (four for a 16-bit cache; twelve, or eight at
//            D = 256, for an FP8 cache) each take 16 keys of every tile and run
//            S^T = K q^T and O^T += V^T P^T on the warp-level tensor cores
//            (the Hq/Hkv grouped query heads are the N = 8 dimension), with an
//            online softmax per head and NO sink.  At the end of an item the
//            warps' (max, sum, O) are merged and one normalised partial
//            (O_s, LSE_s) per query head is written.
//   combine  one warp per (sequence, query head): merges exactly the splits
//            that exist, in split order, and adds the sink once.
// Split-KV decode and the LSE combine: page
// "flashmla-optimization/docs/PATCH_STACK.md", section 3 ("exact small-split
// combine": with <= 32 real splits only the valid LSE lanes are reduced and no
// masked work is built for splits that do not exist; the accumulation order of
// the real splits is kept).  The sink term is the learned sink of page
// "cf-1.com/news/6055759".
//
// Decode moves ~512 bytes of K/V per key per kv head for 8 x 128 x 4 flops, so
// it is bound by HBM bandwidth; the warp-level MMA keeps the arithmetic far
// below that bound without tying up registers in fp32 FMA loops.
#include <math.h>

#include <type_traits>

#include "kernels.h"
#include "ptx.cuh"

namespace attnsink {
namespace {

constexpr int kTK = 64;               // keys per tile (bf16 cache)
constexpr int kConsumerWarps = 4;     // each owns 16 keys of every tile (bf16 cache)

constexpr float kLn2 = 0.6931471805599453f;
enum : int { kWhereFull = 201, kWhereEmpty = 202, kWhereMerge = 203 };

// Workspace layout (each section 256-byte aligned).
struct WsLayout {
  size_t off_nsplit, off_base, off_ctrl, off_lse, off_o, total;
  int max_splits;  // upper bound on the total number of splits
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

WsLayout ws_layout(const DecodeArgs &a) {
  WsLayout w;
  const int per_seq = decode_max_splits_per_seq(a);
  w.max_splits = a.B * per_seq;
  size_t off = 0;
  w.off_nsplit = off;
  off = align256(off + sizeof(int) * a.B);
  w.off_base = off;
  off = align256(off + sizeof(int) * a.B);
  w.off_ctrl = off;                                   // [0] total splits, [1] work counter
  off = align256(off + sizeof(int) * 4);
  w.off_lse = off;
  off = align256(off + sizeof(float) * static_cast<size_t>(w.max_splits) * a.Hq);
  w.off_o = off;
  off = align256(off + sizeof(float) * static_cast<size_t>(w.max_splits) * a.Hq * a.D);
  w.total = off;
  return w;
}

// ------------------------------------------------------------------- plan
__global__ void __launch_bounds__(1024) decode_plan_kernel(const int *seqlens, int B, int Smax,
                                                           int W, int chunk, int align,
                                                           int *nsplit, int *base, int *ctrl) {
  __shared__ int warp_sums[32];
  const int t = threadIdx.x;
  const int per = (B + blockDim.x - 1) / blockDim.x;  // contiguous segment per thread
  const int b0 = t * per;
  int local = 0;
  for (int b = b0; b < min(B, b0 + per); ++b) {
    const int n = min(max(seqlens[b], 0), Smax);
    const int len = n - max(0, n - W) / align * align;
    const int ns = (len + chunk - 1) / chunk;
    nsplit[b] = ns;
    local += ns;
  }
  // block-wide exclusive scan of the per-thread sums
  const int lane = t & 31, wid = t >> 5;
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    const int nw = blockDim.x >> 5;
    int v = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    if (lane < nw) warp_sums[lane] = v;  // inclusive over warps
  }
  __syncthreads();
  int run = incl - local + (wid > 0 ? warp_sums[wid - 1] : 0);
  for (int b = b0; b < min(B, b0 + per); ++b) {
    base[b] = run;
    run += nsplit[b];
  }
  if (t == blockDim.x - 1) {
    ctrl[0] = run;  // total splits
    ctrl[1] = 0;    // work counter for the split kernel
  }
}

// ------------------------------------------------------------------ split
struct SplitParams {
  const __nv_bfloat16 *q;
  int64_t q_sb, q_sh;
  const int *seqlens;
  const int *nsplit, *base, *ctrl;
  int *work_counter;
  float *lse_part, *o_part;
  int B, Smax, Hq, Hkv, G, W, chunk;
  float scale_log2;
  int *status;
  // paged cache (page > 0): position t of sequence b is row t & (page - 1) of
  // pool page block_table[b * bt_s0 + (t >> page_shift)]
  const int *block_table;
  int64_t bt_s0;
  int page, page_shift, max_pages, align;
  // log2 of the key rows R of one K (or V) TMA box: a 16-bit stage holds, per
  // K/V tile, [box][64-channel chunk][row in box][128 bytes] (R = the tile's
  // 64 rows, i.e. [chunk][row], except for pages of 16 or 32 positions, whose
  // box is one page of every chunk)
  int rows_shift;
  // FP8 e4m3 cache: per-kv-head dequantisation scales (key row = k_descale *
  // e4m3 row; v_descale scales the partial output)
  const float *k_descale, *v_descale;
};

struct StageInfo {
  int b, hk, split, key0, nvalid, flags;  // flags: 1 first tile, 2 last tile, 4 end of work
  int nskip;                              // keys [0, nskip) of the tile precede the window
  int pad;
};

// kF8: the cache holds FP8 e4m3 bytes, in 128-byte (128-element) swizzled
// chunks.  Each consumer warp converts its K and V operands to f16 in
// registers straight from the stage (one cvt per pair, exact) and runs the
// MMAs below in f16: q is converted to f16 after a power-of-two scale that
// puts its largest magnitude in [2^13, 2^14) (undone in the softmax scale),
// and P is f16.  Because a 16-byte row unit read by ldmatrix hands each lane
// four consecutive e4m3 values, the contraction index of S^T = K q^T is
// permuted (k = 2t, 2t+1, 2t+8, 2t+9 of a k-step hold d = 4t .. 4t+3 of its
// 16-d unit), and q is loaded in the same order; V goes through
// ldmatrix.trans of byte pairs (keys 2t, 2t+1 at two consecutive d per lane)
// and one byte permute, which orders the d rows of O^T within each 16-d unit
// as 0, 2, .., 14 then 1, 3, .., 15 (the merge writes them back in order).
// An FP8 cache delivers a key in half the bytes, so at D = 128 its tiles are
// 192 keys for 12 consumer warps (128 keys and 8 warps for groups of more
// than 8 heads, whose accumulators need the registers).  The merge at the end
// of an item runs in the stage it has just consumed (one head tile per pass),
// which is released after it; the ring takes all the rest of shared memory.
template <int D, int NT, bool kF8>
struct DCfg {
  // consumer warps: FP8 caches take more warps per scheduler to hide the
  // conversion latency (D = 256: eight, as many as three 64 KB stages and the
  // merge in one stage allow)
  static constexpr int kCW = kF8 ? (D == 128 ? 12 : 8) : kConsumerWarps;
  // FP8 cache, two head tiles: each consumer warp keeps its q fragments in a
  // private slice of shared memory instead of 32 registers, so that twelve
  // consumer warps (four warps per scheduler, 128 registers each) fit
  static constexpr bool kQInSmem = kF8 && NT == 2;
  static constexpr int kTK = 16 * kCW;                    // keys per tile
  static constexpr int kThreads = (kCW + 1) * 32;         // + the producer warp
  static constexpr bool kMergeInStage = kF8;
  static constexpr int kMergePasses = kMergeInStage ? NT : 1;   // head tiles merged one pass at a time
  static constexpr int kChunks = D / 64;                  // 64-element chunks of a bf16 row
  static constexpr int kChunks8 = D / 128;                // 128-element chunks of an FP8 row
  static constexpr int kTileBytes = kTK * D * (kF8 ? 1 : 2);   // one K (or V) tile as stored
  static constexpr int kStageBytes = 2 * kTileBytes;      // K then V
  static constexpr int kMergeBytes = kCW * NT * 8 * D * 4;
  static constexpr int kQBytes = kQInSmem ? kCW * (D / 16) * NT * 32 * 8 : 0;   // [warp][kk][nt][lane] uint2
  static constexpr int kRingBudget = kF8 ? 232448 - 1024 - 2048 - kQBytes : 196608 - kMergeBytes;
  static constexpr int kStages = (kRingBudget / kStageBytes) > 12 ? 12 : (kRingBudget / kStageBytes);
  static constexpr int kMergeOffset = kStages * kStageBytes;   // (16-bit cache only)
  static constexpr int kQOffset = kStages * kStageBytes;       // (kQInSmem only)
  static constexpr int kInfoOffset = kStages * kStageBytes + (kMergeInStage ? 0 : kMergeBytes) + kQBytes;
  static_assert(!kMergeInStage || kCW * (NT / kMergePasses) * 8 * D * 4 <= kStageBytes,
                "one merge pass fits a stage");
  // stage descriptors, full/empty barriers, the consumers' merge barrier,
  // per-warp (max, sum) for the merge, the abort flag; plus 1 KB of slack for
  // aligning the base to 1 KB
  static constexpr int kInfoBytes =
      (kStages * 32 + kStages * 16 + 8 + 2 * kCW * NT * 8 * 4 + 16 + 127) / 128 * 128;
  static constexpr int kSmemBytes = kInfoOffset + kInfoBytes + 1024;
  static_assert(kSmemBytes <= 232448, "shared-memory budget");
  static_assert(!kF8 || kInfoBytes <= 2048, "FP8 ring budget leaves room for the stage info");
  static_assert(!kF8 || D % 128 == 0, "FP8 rows are whole 128-byte chunks");
};

// Four e4m3 values (a 32-bit word, low byte first) to two f16 pairs: the word
// splits into its 16-bit halves, one cvt each; exact (every e4m3 value,
// subnormals included, is a normal f16; NaN stays NaN).
__device__ __forceinline__ uint2 e4m3x4_to_f16x4(uint32_t w) {
  uint2 h;
  asm("{.reg .b16 lo, hi; mov.b32 {lo, hi}, %2; cvt.rn.f16x2.e4m3x2 %0, lo; cvt.rn.f16x2.e4m3x2 %1, hi;}"
      : "=r"(h.x), "=r"(h.y)
      : "r"(w));
  return h;
}

// bf16 pair -> f16 pair times a power of two (exact unless the product falls
// below the f16 normal range).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2_scaled(uint32_t x, float s) {
  const float lo = __uint_as_float(x << 16) * s, hi = __uint_as_float(x & 0xFFFF0000u) * s;
  return pack_f16x2(lo, hi);
}

__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, const WaitCtx &ctx,
                                          int where) {
  const bool r = mbar_wait(bar, parity, ctx, where);
  return __all_sync(0xffffffffu, r);
}

// Before the producer leaves, the copies into the stages it armed have landed:
// the CTA and its shared memory must outlive them, also when the consumers
// gave up early.  `armed` stages were armed; only the last kStages of them
// can still be in flight.  Each wait is bounded by the fixed limit, whatever
// limit the other waits use.
template <int kStages>
__device__ __forceinline__ void drain_stages(uint64_t *full, int armed) {
  for (int x = max(0, armed - kStages); x < armed; ++x) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(&full[x % kStages], static_cast<uint32_t>(x / kStages) & 1u))
      if (globaltimer_ns() - t0 > kWaitLimitNs) break;
  }
}

template <int D, int NT, bool kF8>
__global__ void __launch_bounds__(DCfg<D, NT, kF8>::kThreads, 1)
    decode_split_kernel(const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const SplitParams p) {
  using C = DCfg<D, NT, kF8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  float *merge = reinterpret_cast<float *>(smem + C::kMergeOffset);
  StageInfo *info = reinterpret_cast<StageInfo *>(smem + C::kInfoOffset);
  uint64_t *full = reinterpret_cast<uint64_t *>(info + C::kStages);
  uint64_t *empty = full + C::kStages;
  uint64_t *merge_bar = empty + C::kStages;   // the consumer warps meet here around a merge
  float *merge_m = reinterpret_cast<float *>(merge_bar + 1);   // [4][NT*8]
  float *merge_l = merge_m + C::kCW * NT * 8;               // [4][NT*8]
  int *abort_flag = reinterpret_cast<int *>(merge_l + C::kCW * NT * 8);
  const WaitCtx ctx{abort_flag, p.status, wait_limit_ns(p.status)};

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], C::kCW);
    }
    mbar_init(merge_bar, C::kCW * 32);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == C::kCW) {
    const bool small_pages = !kF8 && p.page != 0 && p.page < C::kTK;
    // -------------------------------------------------------------- producer
    // Contiguous cache, FP8 cache, or pages of at least a tile: one lane
    // issues everything.
    if (!small_pages && lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const int total_items = p.ctrl[0] * p.Hkv;
      int slot = 0;
      bool ok = true;
      auto acquire = [&]() -> int {
        const int s = slot % C::kStages;
        const uint32_t use = static_cast<uint32_t>(slot / C::kStages);
        if (slot >= C::kStages && !mbar_wait(&empty[s], (use & 1u) ^ 1u, ctx, kWhereEmpty))
          ok = false;
        ++slot;
        return s;
      };
      while (ok) {
        const int w = atomicAdd(p.work_counter, 1);
        if (w >= total_items) break;
        const int g = w / p.Hkv, hk = w - g * p.Hkv;
        int lo = 0, hi = p.B - 1;  // last b with base[b] <= g
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (p.base[mid] <= g) lo = mid; else hi = mid - 1;
        }
        const int b = lo;
        const int split = g - p.base[b];
        const int n = min(max(p.seqlens[b], 0), p.Smax);
        const int vis0 = max(0, n - p.W);
        const int ks = vis0 / p.align * p.align + split * p.chunk;
        const int ke = min(n, ks + p.chunk);
        const int nt = (ke - ks + C::kTK - 1) / C::kTK;
        const int nbox = p.page == 0 ? 1 : C::kTK / min(C::kTK, p.page);   // boxes per tile (paged)
        for (int t = 0; ok && t < nt; ++t) {
          // Paged cache: read the tile's page numbers before waiting for a free
          // stage, so that the table reads overlap the wait.
          int blk[4] = {0, 0, 0, 0};
          if (p.page != 0) {
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              if (r >= nbox) break;
              const int lp = (ks + t * C::kTK + r * (C::kTK / nbox)) >> p.page_shift;
              blk[r] = lp < p.max_pages ? p.block_table[static_cast<int64_t>(b) * p.bt_s0 + lp] : -1;
            }
          }
          const int s = acquire();
          if (!ok) break;
          StageInfo &si = info[s];
          si.b = b;
          si.hk = hk;
          si.split = split;
          si.key0 = ks + t * C::kTK;
          si.nvalid = min(C::kTK, ke - si.key0);
          si.nskip = max(0, vis0 - si.key0);
          si.flags = (t == 0 ? 1 : 0) | (t == nt - 1 ? 2 : 0);
          mbar_arrive_expect_tx(&full[s], C::kStageBytes);
          uint8_t *dst = smem + s * C::kStageBytes;
          if (kF8) {
            for (int c = 0; c < C::kChunks8; ++c) {
              tma_load_4d(dst + c * C::kTK * 128, &tmK, &full[s], c * 128, hk, si.key0, b);
              tma_load_4d(dst + C::kTileBytes + c * C::kTK * 128, &tmV, &full[s], c * 128, hk, si.key0, b);
            }
          } else if (p.page == 0) {
            for (int c = 0; c < C::kChunks; ++c) {
              tma_load_4d(dst + c * C::kTK * 128, &tmK, &full[s], c * 64, hk, si.key0, b);
              tma_load_4d(dst + C::kTileBytes + c * C::kTK * 128, &tmV, &full[s], c * 64, hk, si.key0, b);
            }
          } else {
            // key0 is a multiple of 64 here, so each box of min(64, page) rows
            // lies in one page.  A table entry outside the pool (or a page
            // number past the table, for rows beyond the sequence end) loads
            // zero rows: the box is out of range and filled, and it still
            // delivers its bytes.
            const int rows = C::kTK / nbox;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              if (r >= nbox) break;
              const int r0 = r * rows;
              const int slot = (si.key0 + r0) & (p.page - 1);
              for (int c = 0; c < C::kChunks; ++c) {
                tma_load_4d(dst + c * C::kTK * 128 + r0 * 128, &tmK, &full[s], c * 64, hk, slot, blk[r]);
                tma_load_4d(dst + C::kTileBytes + c * C::kTK * 128 + r0 * 128, &tmV, &full[s], c * 64, hk,
                            slot, blk[r]);
              }
            }
          }
        }
      }
      if (ok) {
        const int s = acquire();
        if (ok) {
          info[s].flags = 4;
          mbar_arrive(&full[s]);
        }
      }
      // (a failed acquire took a stage it never armed)
      drain_stages<C::kStages>(full, ok ? slot : slot - 1);
    }
    // Pages smaller than a tile (several pages per tile): the whole warp
    // follows one control flow; lane 0 claims work, waits for free stages and
    // arms their barriers (results shared by shuffle), and the copies of a
    // tile (one per page and K/V) are issued by one lane each.
    if (small_pages) {
      if (lane == 0) {
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
      }
      const int total_items = p.ctrl[0] * p.Hkv;
      int slot = 0;
      bool ok = true;
      auto acquire = [&]() -> int {
        const int s = slot % C::kStages;
        const uint32_t use = static_cast<uint32_t>(slot / C::kStages);
        bool good = true;
        if (lane == 0 && slot >= C::kStages && !mbar_wait(&empty[s], (use & 1u) ^ 1u, ctx, kWhereEmpty))
          good = false;
        ok = ok && __shfl_sync(0xffffffffu, good, 0);
        ++slot;
        return s;
      };
      while (ok) {
        int w = 0;
        if (lane == 0) w = atomicAdd(p.work_counter, 1);
        w = __shfl_sync(0xffffffffu, w, 0);
        if (w >= total_items) break;
        const int g = w / p.Hkv, hk = w - g * p.Hkv;
        int lo = 0, hi = p.B - 1;  // last b with base[b] <= g
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (p.base[mid] <= g) lo = mid; else hi = mid - 1;
        }
        const int b = lo;
        const int split = g - p.base[b];
        const int n = min(max(p.seqlens[b], 0), p.Smax);
        const int vis0 = max(0, n - p.W);
        const int ks = vis0 / p.align * p.align + split * p.chunk;
        const int ke = min(n, ks + p.chunk);
        const int nt = (ke - ks + C::kTK - 1) / C::kTK;
        const int nbox = p.page == 0 ? 1 : C::kTK / min(C::kTK, p.page);   // boxes per tile (paged)
        for (int t = 0; ok && t < nt; ++t) {
          const int key0 = ks + t * C::kTK;
          // Paged cache: lane r < nbox reads box r's page number before the
          // stage wait, so that the table reads overlap it.
          int blk = 0;
          if (p.page != 0 && lane < nbox) {
            const int lp = (key0 + lane * (C::kTK / nbox)) >> p.page_shift;
            blk = lp < p.max_pages ? p.block_table[static_cast<int64_t>(b) * p.bt_s0 + lp] : -1;
          }
          const int s = acquire();
          if (!ok) break;
          uint8_t *dst = smem + s * C::kStageBytes;
          if (lane == 0) {
            StageInfo &si = info[s];
            si.b = b;
            si.hk = hk;
            si.split = split;
            si.key0 = key0;
            si.nvalid = min(C::kTK, ke - key0);
            si.nskip = max(0, vis0 - key0);
            si.flags = (t == 0 ? 1 : 0) | (t == nt - 1 ? 2 : 0);
            mbar_arrive_expect_tx(&full[s], C::kStageBytes);
          }
          __syncwarp();
          if (kF8) {
            if (lane == 0)
              for (int c = 0; c < C::kChunks8; ++c) {
                tma_load_4d(dst + c * C::kTK * 128, &tmK, &full[s], c * 128, hk, key0, b);
                tma_load_4d(dst + C::kTileBytes + c * C::kTK * 128, &tmV, &full[s], c * 128, hk, key0, b);
              }
          } else if (p.page == 0) {
            if (lane == 0)
              for (int c = 0; c < C::kChunks; ++c) {
                tma_load_4d(dst + c * C::kTK * 128, &tmK, &full[s], c * 64, hk, key0, b);
                tma_load_4d(dst + C::kTileBytes + c * C::kTK * 128, &tmV, &full[s], c * 64, hk, key0, b);
              }
          } else {
            // key0 is a multiple of 64 here, so the tile is nbox whole pages.
            // Lane (r, kv) issues page r of K (kv = 0) or V (kv = 1): one box
            // of every 64-channel chunk of the page's rows (5-D page view),
            // at box slot r of the stage layout.  A table entry outside the
            // pool (or a page number past the table, for rows beyond the
            // sequence end) loads zero rows: the box is out of range and
            // filled, and it still delivers its bytes.
            const int r = lane >> 1, kv = lane & 1;
            const int blk_r = __shfl_sync(0xffffffffu, blk, r < nbox ? r : 0);
            if (lane < 2 * nbox)
              tma_load_5d(dst + kv * C::kTileBytes + r * (C::kChunks * 128 * p.page), kv ? &tmV : &tmK,
                          &full[s], 0, 0, 0, hk, blk_r);
          }
        }
      }
      if (ok) {
        const int s = acquire();
        if (ok && lane == 0) {
          info[s].flags = 4;
          mbar_arrive(&full[s]);
        }
      }
      if (lane == 0) drain_stages<C::kStages>(full, ok ? slot : slot - 1);
    }
    __syncwarp();
    return;
  }

  // ------------------------------------------------------------- consumers
  const int g8 = lane >> 2;       // mma "group" (row within an 8-row block)
  const int tig = lane & 3;       // thread in group
  // 16-bit stage: byte offset of a key row within a K/V tile, and of a
  // 64-channel chunk within a box ([box][chunk][row in box][128 bytes]; the
  // row's swizzle phase stays row & 7, as a box holds a multiple of 8 rows)
  const int rs = p.rows_shift;
  auto row_off = [&](int row) -> uint32_t {
    return static_cast<uint32_t>((((row >> rs) * C::kChunks) << (rs + 7)) + ((row & ((1 << rs) - 1)) << 7));
  };
  const uint32_t cstride = 128u << rs;
  const int key_w = warp * 16;    // this warp's 16 keys within a tile
  const int krow = key_w + (lane & 7) + ((lane >> 3) & 1) * 8;   // ldmatrix rows of S^T = K q^T
  const int vrow = key_w + (lane & 7) + (lane >> 4) * 8;         // ldmatrix.trans rows of V^T
  const uint32_t krow_off = row_off(krow), vrow_off = row_off(vrow);
  const uint32_t zrow_off = row_off(key_w + (lane & 15));        // V rows zeroed by lanes l, l + 16
  float sl2 = p.scale_log2;       // (FP8: times the item's key descale)
  float vdesc = 1.f;              // (FP8: the item's value descale)
  // B fragments of q^T, per k-step and head tile (kQInSmem: the item's copy
  // lives in this warp's slice of shared memory between tiles)
  uint32_t qf[C::kQInSmem ? 1 : D / 16][NT][2];
  uint2 *qsm = reinterpret_cast<uint2 *>(smem + C::kQOffset) + warp * (D / 16) * NT * 32 + lane;
  float o[D / 16][NT][4];         // O^T accumulators: [d tile][head tile][frag]
  float m_run[NT][2], l_run[NT][2];
  // The consumer warps meet around each merge through an mbarrier (every
  // consumer thread arrives, then waits for the phase, bounded): a warp that
  // gave up on a wait leaves, and the others' next meeting then runs out
  // instead of waiting for it forever.
  uint32_t merge_phase = 0;
  auto consumers_meet = [&]() -> bool {
    mbar_arrive(merge_bar);
    const bool met = warp_wait(merge_bar, merge_phase & 1u, ctx, kWhereMerge);
    ++merge_phase;
    return met;
  };
  int slot = 0;
  while (true) {
    const int s = slot % C::kStages;
    if (!warp_wait(&full[s], static_cast<uint32_t>(slot / C::kStages) & 1u, ctx, kWhereFull)) break;
    ++slot;
    const StageInfo si = info[s];
    if (si.flags & 4) break;
    const uint32_t kbase = smem_u32(smem + s * C::kStageBytes);
    const uint32_t vbase = kbase + C::kTileBytes;
    if (si.flags & 1) {
      // first tile of a work item: load this kv head's grouped queries
      uint32_t qx[D / 16][NT][2];
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int hl = nt * 8 + g8;
          uint32_t x0 = 0, x1 = 0;
          if (hl < p.G) {
            // 16-bit cache: k = 2t, 2t+1 | 2t+8, 2t+9 of the k-step are d =
            // 16kk + 2t, +1 | +8, +9; FP8 cache: d = 16kk + 4t .. 4t+3
            const __nv_bfloat16 *qr =
                p.q + si.b * p.q_sb + (si.hk * p.G + hl) * p.q_sh + kk * 16 + (kF8 ? 4 : 2) * tig;
            x0 = *reinterpret_cast<const uint32_t *>(qr);
            x1 = *reinterpret_cast<const uint32_t *>(qr + (kF8 ? 2 : 8));
          }
          qx[kk][nt][0] = x0;
          qx[kk][nt][1] = x1;
        }
#pragma unroll
      for (int dm = 0; dm < D / 16; ++dm)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int f = 0; f < 4; ++f) o[dm][nt][f] = 0.f;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        m_run[nt][0] = m_run[nt][1] = -INFINITY;
        l_run[nt][0] = l_run[nt][1] = 0.f;
      }
      if constexpr (kF8) {
        // q to f16 with a power-of-two scale 2^e that puts max|q| in
        // [2^13, 2^14): exact for every q element above max|q| * 2^-27;
        // 2^-e then joins the softmax scale with the key descale
        float mx = 0.f;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int f = 0; f < 2; ++f) {
              const uint32_t x = qx[kk][nt][f];
              mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(x << 16)), fabsf(__uint_as_float(x & 0xFFFF0000u))));
            }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        int e = 0;
        if (mx > 0.f && mx < INFINITY) e = 13 - ilogbf(mx);
        const float qs = ldexpf(1.f, e);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int f = 0; f < 2; ++f) qx[kk][nt][f] = bf16x2_to_f16x2_scaled(qx[kk][nt][f], qs);
        sl2 = p.scale_log2 * p.k_descale[si.hk] * ldexpf(1.f, -e);
        vdesc = p.v_descale[si.hk];
      }
      if constexpr (C::kQInSmem) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) qsm[(kk * NT + nt) * 32] = make_uint2(qx[kk][nt][0], qx[kk][nt][1]);
        __syncwarp();
      } else {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            qf[kk][nt][0] = qx[kk][nt][0];
            qf[kk][nt][1] = qx[kk][nt][1];
          }
      }
    }
    // Keys past the end of the split, and (paged cache) keys before the
    // window, are masked; their cache rows may hold anything (NaN included),
    // so their V rows are zeroed in shared memory before P.V reads them.
    if (!kF8 && (si.nvalid < key_w + 16 || si.nskip > key_w)) {
      const int kidx = key_w + (lane & 15);
      if (kidx >= si.nvalid || kidx < si.nskip) {
        for (int c = 0; c < C::kChunks; ++c) {
          uint8_t *row = smem + s * C::kStageBytes + C::kTileBytes + c * cstride + zrow_off;
          const int half = lane >> 4;
#pragma unroll
          for (int u = 0; u < 4; ++u)
            *reinterpret_cast<uint4 *>(row + (half * 4 + u) * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      __syncwarp();
    }
    // ---- S^T[16 keys x 8*NT heads] = K_w q^T ----
    float sacc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int f = 0; f < 4; ++f) sacc[nt][f] = 0.f;
    if constexpr (kF8) {
      // ldmatrix of e4m3 bytes: matrices (keys 0-7 | 8-15) x (unit u | u+1)
      // of a 128-byte chunk; lane (g, t) receives d = 16u + 4t .. 4t+3 of
      // keys g and g+8, i.e. the A fragments of k-steps u and u+1 once
      // converted
      const int r = lane & 7;
      const int krow8 = key_w + r + ((lane >> 3) & 1) * 8;   // krow8 & 7 == r
#pragma unroll
      for (int c8 = 0; c8 < C::kChunks8; ++c8)
#pragma unroll
        for (int up = 0; up < 4; ++up) {
          const int unit = 2 * up + (lane >> 4);
          const uint32_t addr = kbase + c8 * (C::kTK * 128) + krow8 * 128 + ((unit ^ r) << 4);
          uint32_t w0, w1, w2, w3;
          ldmatrix_x4(addr, w0, w1, w2, w3);
          const uint2 k0 = e4m3x4_to_f16x4(w0), k1 = e4m3x4_to_f16x4(w1);
          const uint2 k2 = e4m3x4_to_f16x4(w2), k3 = e4m3x4_to_f16x4(w3);
          const int kk = c8 * 8 + 2 * up;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            uint2 qa, qb;
            if constexpr (C::kQInSmem) {
              qa = qsm[(kk * NT + nt) * 32];
              qb = qsm[((kk + 1) * NT + nt) * 32];
            } else {
              qa = make_uint2(qf[kk][nt][0], qf[kk][nt][1]);
              qb = make_uint2(qf[kk + 1][nt][0], qf[kk + 1][nt][1]);
            }
            mma_f16_16816(sacc[nt], k0.x, k1.x, k0.y, k1.y, qa.x, qa.y);
            mma_f16_16816(sacc[nt], k2.x, k3.x, k2.y, k3.y, qb.x, qb.y);
          }
        }
    } else {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int unit = 2 * (kk & 3) + (lane >> 4);
        const uint32_t addr = kbase + (kk >> 2) * cstride + krow_off + ((unit ^ (krow & 7)) << 4);
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(addr, a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          mma_bf16_16816(sacc[nt], a0, a1, a2, a3, qf[kk][nt][0], qf[kk][nt][1]);
      }
    }
    // ---- online softmax per head (no sink here) ----
    const int kv0 = key_w + g8, kv1 = key_w + g8 + 8;
    const bool v0 = kv0 >= si.nskip && kv0 < si.nvalid, v1 = kv1 >= si.nskip && kv1 < si.nvalid;
    uint32_t pb[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float x[4];
      x[0] = v0 ? sacc[nt][0] * sl2 : -INFINITY;  // key g,   head 2tig
      x[1] = v0 ? sacc[nt][1] * sl2 : -INFINITY;  // key g,   head 2tig+1
      x[2] = v1 ? sacc[nt][2] * sl2 : -INFINITY;  // key g+8, head 2tig
      x[3] = v1 ? sacc[nt][3] * sl2 : -INFINITY;  // key g+8, head 2tig+1
      float mx0 = fmaxf(x[0], x[2]), mx1 = fmaxf(x[1], x[3]);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
      }
      const float n0 = fmaxf(m_run[nt][0], mx0), n1 = fmaxf(m_run[nt][1], mx1);
      const float a0 = (n0 == -INFINITY) ? 1.f : ex2_approx(m_run[nt][0] - n0);
      const float a1 = (n1 == -INFINITY) ? 1.f : ex2_approx(m_run[nt][1] - n1);
      m_run[nt][0] = n0;
      m_run[nt][1] = n1;
      const float u0 = (n0 == -INFINITY) ? 0.f : n0, u1 = (n1 == -INFINITY) ? 0.f : n1;
      const float p0 = ex2_approx(x[0] - u0), p1 = ex2_approx(x[1] - u1);
      const float p2 = ex2_approx(x[2] - u0), p3 = ex2_approx(x[3] - u1);
      l_run[nt][0] = l_run[nt][0] * a0 + p0 + p2;
      l_run[nt][1] = l_run[nt][1] * a1 + p1 + p3;
      if (a0 != 1.f || a1 != 1.f) {
#pragma unroll
        for (int dm = 0; dm < D / 16; ++dm) {
          o[dm][nt][0] *= a0;
          o[dm][nt][1] *= a1;
          o[dm][nt][2] *= a0;
          o[dm][nt][3] *= a1;
        }
      }
      // P^T fragments (key rows, head columns) -> transposed into the
      // B-operand layout of O^T += V^T P^T.
      pb[nt][0] = movmatrix_trans(kF8 ? pack_f16x2(p0, p1) : pack_bf16x2(p0, p1));
      pb[nt][1] = movmatrix_trans(kF8 ? pack_f16x2(p2, p3) : pack_bf16x2(p2, p3));
    }
    // ---- O^T[D x 8*NT] += V_w^T P^T ----
    if constexpr (kF8) {
      // ldmatrix.trans of e4m3 bytes taken as 16-bit pairs: matrices (keys
      // 0-7 | 8-15) x (unit u | u+1); lane (g, t) receives keys 2t, 2t+1 (or
      // 2t+8, 2t+9) at d = 16u + 2g and 2g + 1, which one byte permute turns
      // into key pairs per d: O^T rows g and g+8 of m-tile u are d = 16u + 2g
      // and 16u + 2g + 1.  Rows outside [nskip, nvalid) may hold NaN bytes:
      // on the tiles that have any, they are zeroed in the registers.
      const int r = lane & 7;
      const int vrow8 = key_w + r + ((lane >> 3) & 1) * 8;   // vrow8 & 7 == r
      auto pv = [&](auto masked) {
        uint32_t mlo = 0xFFFFFFFFu, mhi = 0xFFFFFFFFu;
        if constexpr (decltype(masked)::value) {
          const int ka = key_w + 2 * tig;
          auto ok = [&](int k) { return k >= si.nskip && k < si.nvalid; };
          mlo = (ok(ka) ? 0x0000FFFFu : 0u) | (ok(ka + 1) ? 0xFFFF0000u : 0u);
          mhi = (ok(ka + 8) ? 0x0000FFFFu : 0u) | (ok(ka + 9) ? 0xFFFF0000u : 0u);
        }
#pragma unroll
        for (int c8 = 0; c8 < C::kChunks8; ++c8)
#pragma unroll
          for (int up = 0; up < 4; ++up) {
            const int unit = 2 * up + (lane >> 4);
            const uint32_t addr = vbase + c8 * (C::kTK * 128) + vrow8 * 128 + ((unit ^ r) << 4);
            uint32_t w0, w1, w2, w3;
            ldmatrix_x4_trans(addr, w0, w1, w2, w3);
            if constexpr (decltype(masked)::value) {
              w0 &= mlo;
              w1 &= mhi;
              w2 &= mlo;
              w3 &= mhi;
            }
            const uint2 v0 = e4m3x4_to_f16x4(__byte_perm(w0, 0u, 0x3120));
            const uint2 v1 = e4m3x4_to_f16x4(__byte_perm(w1, 0u, 0x3120));
            const uint2 v2 = e4m3x4_to_f16x4(__byte_perm(w2, 0u, 0x3120));
            const uint2 v3 = e4m3x4_to_f16x4(__byte_perm(w3, 0u, 0x3120));
            const int dm = c8 * 8 + 2 * up;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              mma_f16_16816(o[dm][nt], v0.x, v0.y, v1.x, v1.y, pb[nt][0], pb[nt][1]);
              mma_f16_16816(o[dm + 1][nt], v2.x, v2.y, v3.x, v3.y, pb[nt][0], pb[nt][1]);
            }
          }
      };
      if (si.nskip <= key_w && si.nvalid >= key_w + 16)
        pv(std::false_type{});
      else
        pv(std::true_type{});
    } else {
#pragma unroll
      for (int dm = 0; dm < D / 16; ++dm) {
        const int unit = 2 * (dm & 3) + ((lane >> 3) & 1);
        const uint32_t addr = vbase + (dm >> 2) * cstride + vrow_off + ((unit ^ (vrow & 7)) << 4);
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4_trans(addr, a0, a1, a2, a3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          mma_bf16_16816(o[dm][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
      }
    }
    // release the stage (generic-proxy writes above are ordered before the
    // next TMA write into it); an FP8 stage is only read here, and the last
    // one of an item is released after the merge that reuses it
    if constexpr (!kF8) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    } else if (!(si.flags & 2)) {
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }

    if (si.flags & 2) {
      // ---- merge the consumer warps' partial states and write (O_s, LSE_s) ----
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float l = l_run[nt][e];
#pragma unroll
          for (int off = 4; off < 32; off <<= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
          l_run[nt][e] = l;
        }
      // previous merge fully read (FP8: and every warp done with this stage)
      if (!consumers_meet()) return;
      if (g8 == 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            merge_m[warp * NT * 8 + nt * 8 + 2 * tig + e] = m_run[nt][e];
            merge_l[warp * NT * 8 + nt * 8 + 2 * tig + e] = l_run[nt][e];
          }
      }
      // the per-warp O^T partials go through the merge buffer (FP8: the
      // stage just consumed), kTP head tiles per pass
      constexpr int kTP = NT / C::kMergePasses;
      float *mbuf = C::kMergeInStage ? reinterpret_cast<float *>(smem + s * C::kStageBytes) : merge;
      const int tid = threadIdx.x;  // 0 .. consumer threads - 1
      const int gsplit = p.base[si.b] + si.split;
#pragma unroll
      for (int ps = 0; ps < C::kMergePasses; ++ps) {
        if (ps > 0 && !consumers_meet()) return;   // previous pass fully read
        float *mw = mbuf + warp * (kTP * 8 * D);  // [head of the pass][d]
#pragma unroll
        for (int dm = 0; dm < D / 16; ++dm)
#pragma unroll
          for (int j = 0; j < kTP; ++j) {
            const int nt = ps * kTP + j;
            const int hh = j * 8 + 2 * tig;
            const int d0 = kF8 ? dm * 16 + 2 * g8 : dm * 16 + g8;  // O^T row g
            const int d1 = kF8 ? d0 + 1 : d0 + 8;                                       // O^T row g + 8
            mw[hh * D + d0] = o[dm][nt][0];
            mw[(hh + 1) * D + d0] = o[dm][nt][1];
            mw[hh * D + d1] = o[dm][nt][2];
            mw[(hh + 1) * D + d1] = o[dm][nt][3];
          }
        if (!consumers_meet()) return;
        const int h0 = ps * kTP * 8;
        const int nh = min(p.G - h0, kTP * 8);
        for (int e = tid; e < nh * D; e += C::kCW * 32) {
          const int hl = e / D, d = e - hl * D, hh = h0 + hl;
          float M = -INFINITY;
#pragma unroll
          for (int w = 0; w < C::kCW; ++w) M = fmaxf(M, merge_m[w * NT * 8 + hh]);
          float num = 0.f, den = 0.f;
#pragma unroll
          for (int w = 0; w < C::kCW; ++w) {
            const float mw_ = merge_m[w * NT * 8 + hh];
            const float f = (mw_ == -INFINITY) ? 0.f : ex2_approx(mw_ - M);
            num += f * mbuf[w * (kTP * 8 * D) + hl * D + d];
            den += f * merge_l[w * NT * 8 + hh];
          }
          const int hq = si.hk * p.G + hh;
          const size_t row = static_cast<size_t>(gsplit) * p.Hq + hq;
          p.o_part[row * D + d] = num / den * vdesc;
          if (d == 0) p.lse_part[row] = (M + log2f(den)) * kLn2;
        }
      }
      if constexpr (C::kMergeInStage) {
        // every reader of the merge is done; its generic writes are ordered
        // before the next TMA write into the stage
        if (!consumers_meet()) return;
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
    }
  }
}

// ---------------------------------------------------------------- combine
template <int D>
__global__ void __launch_bounds__(128) decode_combine_kernel(const int *nsplit, const int *base,
                                                             const float *lse_part,
                                                             const float *o_part,
                                                             const float *sinks,
                                                             __nv_bfloat16 *out, int64_t o_sb,
                                                             int64_t o_sh, int B, int Hq) {
  constexpr int DPL = D / 32;
  const int wg = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wg >= B * Hq) return;
  const int b = wg / Hq, hq = wg - b * Hq;
  const int ns = nsplit[b];
  const int sb = base[b];
  const float sink = sinks[hq];
  float acc[DPL];
#pragma unroll
  for (int t = 0; t < DPL; ++t) acc[t] = 0.f;
  float M = sink, den;
  if (ns <= 32) {
    // Exact small-split path: only the lanes of splits that exist hold an LSE.
    const float ls = lane < ns ? lse_part[static_cast<size_t>(sb + lane) * Hq + hq] : -INFINITY;
    float mx = ls;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    M = fmaxf(M, mx);
    const float w = lane < ns ? __expf(ls - M) : 0.f;
    float sw = w;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sw += __shfl_xor_sync(0xffffffffu, sw, off);
    den = sw + ((sink == -INFINITY) ? 0.f : __expf(sink - M));
    for (int s = 0; s < ns; ++s) {  // split order 0, 1, 2, ...
      const float ws = __shfl_sync(0xffffffffu, w, s);
      const float *op = o_part + (static_cast<size_t>(sb + s) * Hq + hq) * D;
#pragma unroll
      for (int t = 0; t < DPL; ++t) acc[t] = fmaf(ws, op[lane + 32 * t], acc[t]);
    }
  } else {
    // General path for more than 32 splits (same arithmetic, chunked).
    for (int s0 = 0; s0 < ns; s0 += 32) {
      const float ls = s0 + lane < ns ? lse_part[static_cast<size_t>(sb + s0 + lane) * Hq + hq] : -INFINITY;
      float mx = ls;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      M = fmaxf(M, mx);
    }
    float sw = 0.f;
    for (int s0 = 0; s0 < ns; s0 += 32) {
      const float ls = s0 + lane < ns ? lse_part[static_cast<size_t>(sb + s0 + lane) * Hq + hq] : -INFINITY;
      const float w = s0 + lane < ns ? __expf(ls - M) : 0.f;
      float t_ = w;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) t_ += __shfl_xor_sync(0xffffffffu, t_, off);
      sw += t_;
      const int cnt = min(32, ns - s0);
      for (int s = 0; s < cnt; ++s) {
        const float ws = __shfl_sync(0xffffffffu, w, s);
        const float *op = o_part + (static_cast<size_t>(sb + s0 + s) * Hq + hq) * D;
#pragma unroll
        for (int t = 0; t < DPL; ++t) acc[t] = fmaf(ws, op[lane + 32 * t], acc[t]);
      }
    }
    den = sw + ((sink == -INFINITY) ? 0.f : __expf(sink - M));
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  __nv_bfloat16 *orow = out + b * o_sb + hq * o_sh;
#pragma unroll
  for (int t = 0; t < DPL; ++t) orow[lane + 32 * t] = __float2bfloat16_rn(acc[t] * inv);
}

template <int D, int NT, bool kF8>
cudaError_t launch_split(const DecodeArgs &a, const WsLayout &w, uint8_t *ws, cudaStream_t stream) {
  using C = DCfg<D, NT, kF8>;
  alignas(64) CUtensorMap mk, mv;
  cudaError_t e;
  if (kF8) {
    if ((e = make_tma_bshd(&mk, a.kc, a.B, a.Smax, a.Hkv, D, a.kc_s, C::kTK, 1)) != cudaSuccess) return e;
    if ((e = make_tma_bshd(&mv, a.vc, a.B, a.Smax, a.Hkv, D, a.vc_s, C::kTK, 1)) != cudaSuccess) return e;
  } else if (a.page == 0) {
    if ((e = make_tma_bshd(&mk, a.kc, a.B, a.Smax, a.Hkv, D, a.kc_s, C::kTK)) != cudaSuccess) return e;
    if ((e = make_tma_bshd(&mv, a.vc, a.B, a.Smax, a.Hkv, D, a.vc_s, C::kTK)) != cudaSuccess) return e;
  } else if (a.page < C::kTK) {
    // one box per page (every chunk): the 5-D page view
    if ((e = make_tma_pages5d(&mk, a.kc, a.npages, a.page, a.Hkv, D, a.kc_s)) != cudaSuccess) return e;
    if ((e = make_tma_pages5d(&mv, a.vc, a.npages, a.page, a.Hkv, D, a.vc_s)) != cudaSuccess) return e;
  } else {
    if ((e = make_tma_bshd(&mk, a.kc, a.npages, a.page, a.Hkv, D, a.kc_s, C::kTK)) != cudaSuccess) return e;
    if ((e = make_tma_bshd(&mv, a.vc, a.npages, a.page, a.Hkv, D, a.vc_s, C::kTK)) != cudaSuccess) return e;
  }
  SplitParams p;
  p.q = static_cast<const __nv_bfloat16 *>(a.q);
  p.q_sb = a.q_s[0];
  p.q_sh = a.q_s[1];
  p.seqlens = a.seqlens;
  p.nsplit = reinterpret_cast<const int *>(ws + w.off_nsplit);
  p.base = reinterpret_cast<const int *>(ws + w.off_base);
  p.ctrl = reinterpret_cast<const int *>(ws + w.off_ctrl);
  p.work_counter = reinterpret_cast<int *>(ws + w.off_ctrl) + 1;
  p.lse_part = reinterpret_cast<float *>(ws + w.off_lse);
  p.o_part = reinterpret_cast<float *>(ws + w.off_o);
  p.B = a.B;
  p.Smax = a.Smax;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.G = a.Hq / a.Hkv;
  p.W = a.W;
  p.chunk = a.chunk;
  p.scale_log2 = static_cast<float>(static_cast<double>(a.scale) * 1.4426950408889634);
  p.status = a.status;
  p.block_table = a.block_table;
  p.bt_s0 = a.bt_s0;
  p.page = a.page;
  p.page_shift = 0;
  while (a.page > 0 && (1 << p.page_shift) < a.page) ++p.page_shift;
  p.max_pages = a.max_pages;
  p.align = a.page > 0 ? C::kTK : 1;
  p.rows_shift = 0;
  if (!kF8) {
    const int rows = (a.page != 0 && a.page < C::kTK) ? a.page : C::kTK;
    while ((1 << p.rows_shift) < rows) ++p.rows_shift;
  }
  p.k_descale = a.k_descale;
  p.v_descale = a.v_descale;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const long long items = static_cast<long long>(w.max_splits) * a.Hkv;
  const int grid = static_cast<int>(items < sms ? items : sms);
  if (grid <= 0) return cudaSuccess;
  auto kern = decode_split_kernel<D, NT, kF8>;
  if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes)) !=
      cudaSuccess)
    return e;
  kern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(mk, mv, p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_combine(const DecodeArgs &a, const WsLayout &w, uint8_t *ws, cudaStream_t stream) {
  const long long warps = static_cast<long long>(a.B) * a.Hq;
  const int blocks = static_cast<int>((warps * 32 + 127) / 128);
  decode_combine_kernel<D><<<blocks, 128, 0, stream>>>(
      reinterpret_cast<const int *>(ws + w.off_nsplit), reinterpret_cast<const int *>(ws + w.off_base),
      reinterpret_cast<const float *>(ws + w.off_lse), reinterpret_cast<const float *>(ws + w.off_o),
      a.sinks, static_cast<__nv_bfloat16 *>(a.out), a.o_s[0], a.o_s[1], a.B, a.Hq);
  return cudaGetLastError();
}

}  // namespace

int decode_max_splits_per_seq(const DecodeArgs &a) {
  // a paged cache's split range starts up to 63 keys before the window
  const long long vis = (a.W < a.Smax ? a.W : a.Smax) + (a.page > 0 ? kTK - 1 : 0);
  return static_cast<int>((vis + a.chunk - 1) / a.chunk);
}

int decode_tile_keys(const DecodeArgs &a) {
  if (!a.fp8 || a.Hkv <= 0) return kTK;
  if (a.D == 128) return a.Hq / a.Hkv <= 8 ? DCfg<128, 1, true>::kTK : DCfg<128, 2, true>::kTK;
  return DCfg<256, 1, true>::kTK;
}

size_t decode_workspace_bytes(const DecodeArgs &a) { return ws_layout(a).total; }

cudaError_t launch_decode(const DecodeArgs &a, void *workspace, cudaStream_t stream) {
  const WsLayout w = ws_layout(a);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  decode_plan_kernel<<<1, 1024, 0, stream>>>(a.seqlens, a.B, a.Smax, a.W, a.chunk,
                                             a.page > 0 ? kTK : 1,
                                             reinterpret_cast<int *>(ws + w.off_nsplit),
                                             reinterpret_cast<int *>(ws + w.off_base),
                                             reinterpret_cast<int *>(ws + w.off_ctrl));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int G = a.Hq / a.Hkv;
  switch (a.D) {
    case 64:
      e = a.fp8 ? cudaErrorInvalidValue
                : (G <= 8 ? launch_split<64, 1, false>(a, w, ws, stream) : launch_split<64, 2, false>(a, w, ws, stream));
      break;
    case 128:
      if (a.fp8)
        e = G <= 8 ? launch_split<128, 1, true>(a, w, ws, stream) : launch_split<128, 2, true>(a, w, ws, stream);
      else
        e = G <= 8 ? launch_split<128, 1, false>(a, w, ws, stream) : launch_split<128, 2, false>(a, w, ws, stream);
      break;
    case 256:
      if (G > 8) e = cudaErrorInvalidValue;
      else e = a.fp8 ? launch_split<256, 1, true>(a, w, ws, stream) : launch_split<256, 1, false>(a, w, ws, stream);
      break;
    default: e = cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  switch (a.D) {
    case 64: return launch_combine<64>(a, w, ws, stream);
    case 128: return launch_combine<128>(a, w, ws, stream);
    case 256: return launch_combine<256>(a, w, ws, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace attnsink
