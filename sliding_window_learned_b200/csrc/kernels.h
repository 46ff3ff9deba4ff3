// kernels.h -- host-side interface between the C ABI (api.cu) and the kernel
// launchers.  Arguments arrive here already validated; strides are in
// elements and the innermost dimension of every tensor is contiguous.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace attnsink {

// Prefill forward: q/out [B,L,Hq,D], k/v [B,L,Hkv,D] (bf16), sinks [Hq] f32,
// lse [B,Hq,L] f32 or null.
struct FwdArgs {
  const void *q, *k, *v;
  const float *sinks;
  void *out;
  float *lse;
  int B, L, Hq, Hkv, D, W;
  float scale;
  int64_t q_s[3], k_s[3], v_s[3], o_s[3];  // strides of dims 0..2
  int64_t lse_s[2];                        // strides of dims 0..1
  int *status;                             // device status word (2 ints)
  // Packed variable-length sequences: q/out [T,Hq,D], k/v [T,Hkv,D] viewed as
  // one batch slice (strides of dim 0 = T * row stride), sequence b is rows
  // cu_seqlens[b] .. cu_seqlens[b+1]-1 (device int32), B = number of
  // sequences, L = an upper bound on their lengths, lse [Hq, T] (lse_s[1] =
  // head stride).  Null: the [B, L] batch above.
  const int *cu_seqlens = nullptr;
  int T = 0;
  // Largest content logit per (batch, query head): [B, Hq] f32 (row stride
  // ml_sb), batched inputs only; null: not computed.
  float *max_logit = nullptr;
  int64_t ml_sb = 0;
};

// Decode: q/out [B,Hq,D], caches [B,Smax,Hkv,D] (bf16), seqlens [B] int32
// (device), sinks [Hq] f32.  With page > 0 the caches are page pools
// [npages, page, Hkv, D] instead: position t of sequence b is row t % page of
// pool page block_table[b * bt_s0 + t / page] (device int32), and
// Smax = max_pages * page.
struct DecodeArgs {
  const void *q, *kc, *vc;
  const int *seqlens;
  const float *sinks;
  void *out;
  int B, Smax, Hq, Hkv, D, W;
  float scale;
  int chunk;                               // keys per split (multiple of 64)
  int64_t q_s[2], kc_s[3], vc_s[3], o_s[2];
  int *status;
  const int *block_table = nullptr;        // paged cache only
  int64_t bt_s0 = 0;
  int page = 0;                            // 0: contiguous cache; else a power of two >= 16
  int npages = 0, max_pages = 0;
  // FP8 e4m3 cache (contiguous only): per-kv-head dequantisation scales
  bool fp8 = false;
  const float *k_descale = nullptr, *v_descale = nullptr;
};

// Backward: q/dq/dout/o [B,L,Hq,D], k/v/dk/dv [B,L,Hkv,D] (bf16; o bf16 or
// f32), lse [B,Hq,L] f32 from the forward, sinks [Hq] f32, dsink [Hq] f32.
struct BwdArgs {
  const void *q, *k, *v, *o, *dout;
  const float *lse, *sinks;
  void *dq, *dk, *dv;
  float *dsink;
  int B, L, Hq, Hkv, D, W;
  float scale;
  bool o_f32;
  int64_t q_s[3], k_s[3], v_s[3], o_s[3], do_s[3], dq_s[3], dk_s[3], dv_s[3], lse_s[2];
  int *status;                             // device status word (2 ints)
};
size_t bwd_workspace_bytes(const BwdArgs &a);
cudaError_t launch_bwd(const BwdArgs &a, void *workspace, cudaStream_t stream);
// The tcgen05 main pass of the backward (D = 64 or 128): dQ, dK, dV summed in
// fp32 workspaces ([B, L, Hq, D], [B, L, Hkv, D], zeroed by the caller) from
// Dsum ([B, Hq, L]).
cudaError_t launch_bwd_main_tc(const BwdArgs &a, const float *dsum, float *dq_acc, float *dk_acc, float *dv_acc,
                               cudaStream_t stream);

// Bytes of stream-ordered workspace one decode call needs (256-byte aligned
// sections: plan, partial LSEs, partial outputs).
size_t decode_workspace_bytes(const DecodeArgs &a);
// Upper bound on the number of splits of one sequence for these arguments.
int decode_max_splits_per_seq(const DecodeArgs &a);
// Keys per K/V tile of the split kernel that runs for these arguments (D, the
// group size Hq/Hkv and the cache type fix it).
int decode_tile_keys(const DecodeArgs &a);

cudaError_t launch_fwd_tc(const FwdArgs &a, cudaStream_t stream);
// Sets every entry of a [B, Hq] max-logit output to -inf.
cudaError_t launch_max_logit_init(float *ml, int64_t sb, int B, int Hq, cudaStream_t stream);
cudaError_t launch_fwd_cudacore(const FwdArgs &a, cudaStream_t stream);
cudaError_t launch_decode(const DecodeArgs &a, void *workspace, cudaStream_t stream);

// Builds a 4-D TMA descriptor for a [d3,d2,d1,d0] bf16 tensor (d0 innermost,
// contiguous) with 128-byte swizzle and a box of {64, 1, box_rows, 1}, i.e.
// box_rows consecutive positions of one head and 64 of its channels.
// Returns cudaErrorInvalidValue if the driver rejects the description.
// elem_bytes = 1 describes a byte tensor (FP8) instead, with a box of
// {128, 1, box_rows, 1}: 128 one-byte elements per 128-byte swizzled row.
// elem_bytes = 4 describes an f32 tensor with whole rows per box
// ({d0, 1, box_rows, 1}, d0 <= 256, no swizzle), for bulk reductions.
cudaError_t make_tma_bshd(void *map_out, const void *base, int64_t d3, int64_t d2, int64_t d1,
                          int64_t d0, const int64_t strides_el[3], int box_rows, int elem_bytes = 2);
// TMA descriptor of a bf16 page pool [npages, page, H, D] (element strides of
// the first three dimensions in strides_el; the last one contiguous) as 5-D
// (64 channels, position in page, 64-channel chunk, head, page) with 128-byte
// swizzle, whose box {64, page, D/64, 1, 1} is one page of one head, every
// chunk: in shared memory [chunk][position][128 bytes].  D a multiple of 64,
// page <= 256.  Returns cudaErrorInvalidValue if the driver rejects it.
cudaError_t make_tma_pages5d(void *map_out, const void *base, int64_t npages, int64_t page, int64_t H,
                             int64_t D, const int64_t strides_el[3]);

}  // namespace attnsink
