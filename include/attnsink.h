/*
 * attnsink.h -- C ABI of libattnsink.so: exact causal sliding-window attention
 * with one learned sink logit per head, and its split-KV decode, for NVIDIA
 * B200 (sm_100a).
 *
 * The operation (page "cf-1.com/news/6055759", section "why it must change:
 * Flint's learned sink"): every query attends to the W most recent keys of its
 * sequence, itself included, and a per-head scalar sink logit joins the softmax
 * denominator as a virtual anchor without a value row.  For query row i of
 * head h, with kv head hk = h / (Hq/Hkv) and visible keys
 * V(i) = { j : max(0, i-W+1) <= j <= i }:
 *
 *   s_j   = scale * <q_i, k_j>
 *   O_i   = sum_{j in V(i)} e^{s_j} v_j / ( sum_{j in V(i)} e^{s_j} + e^{sink_h} )
 *   LSE_i = ln( sum_{j in V(i)} e^{s_j} + e^{sink_h} )
 *
 * The sink is in logit units after scaling (it is not multiplied by scale).
 * Same page, section "fix 2: sink normalisation": the kernels rebase the running
 * maximum on the sink so that no exponent is positive, whichever side dominates.
 *
 * Conventions for every entry point:
 *  - All tensors are described by attn_tensor: a DEVICE pointer, a dtype, and
 *    shape/stride in elements.  The innermost dimension must have stride 1;
 *    every other stride of a bf16 tensor must be a positive multiple of 8
 *    elements (16 bytes) and every base pointer 16-byte aligned.
 *  - The caller owns every buffer.  The library keeps no pointer after a call
 *    returns.  Launches go to `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and are stream-ordered: no call synchronises the host.
 *  - Calls never abort.  They return ATTN_OK or a negative attn_status code.
 *    Argument errors are detected on the host before anything is launched; a
 *    one-line description of the last error on the calling thread is available
 *    from attn_sink_last_error().
 *  - Device-side waits are bounded.  A wait that runs out records
 *    ATTN_ETIMEOUT in a device status word and the kernel returns early;
 *    attn_sink_get_status() reads and clears that word.
 *  - Per device, the library looks up the device addresses of its own
 *    device-side objects (the status word, the no-allocation scratch array)
 *    once, and keeps its workspace pool and tensor-map cache for the life of
 *    the process.  They belong to the device's primary context: do not use
 *    the library on a device after cudaDeviceReset() (or any other teardown
 *    of that primary context) in the same process.
 */
#ifndef ATTNSINK_H
#define ATTNSINK_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum attn_dtype {
    ATTN_DTYPE_BF16 = 1,
    ATTN_DTYPE_F32 = 2,
    ATTN_DTYPE_I32 = 3,
    ATTN_DTYPE_E4M3 = 4   /* FP8: 1 sign, 4 exponent (bias 7), 3 mantissa bits */
};

typedef struct attn_tensor {
    void *data;        /* device pointer (16-byte aligned)                  */
    int32_t dtype;     /* enum attn_dtype                                    */
    int32_t ndim;      /* number of valid entries in shape/stride            */
    int64_t shape[4];
    int64_t stride[4]; /* in elements                                        */
} attn_tensor;

enum attn_status {
    ATTN_OK = 0,
    ATTN_EINVAL = -1,       /* bad shape, dtype, stride, alignment or value   */
    ATTN_EUNSUPPORTED = -2, /* valid but not implemented (e.g. head dim)      */
    ATTN_ECUDA = -3,        /* a CUDA runtime call failed                     */
    ATTN_ENOMEM = -4,       /* stream-ordered workspace allocation failed     */
    ATTN_ETIMEOUT = -5      /* a device-side bounded wait ran out             */
};

/*
 * Prefill forward (page "cf-1.com/news/6055759": learned sink, fix 2).
 *
 *   q      [B, L, Hq, D]  bf16
 *   k, v   [B, L, Hkv, D] bf16, Hq % Hkv == 0
 *   sinks  [Hq]           f32; finite or -inf (-inf = no sink).  +inf or NaN
 *                         give an undefined result.
 *   window W >= 1: number of visible keys including the query's own position;
 *          any W >= L is full causal attention.
 *   scale  softmax scale applied to q.k (typically 1/sqrt(D)); finite, > 0.
 *   out    [B, L, Hq, D]  bf16, written completely (round to nearest even).
 *   lse    [B, Hq, L]     f32 natural-log normaliser including the sink, or
 *                         NULL.  The innermost stride must be 1.
 * Supported head dims D: 64, 128, 256.  L = 0 or B = 0 is a no-op.
 * Runs on the tcgen05/TMEM tensor-core kernel.
 */
int attn_sink_fwd(const attn_tensor *q, const attn_tensor *k, const attn_tensor *v,
                  const attn_tensor *sinks, int32_t window, float scale,
                  attn_tensor *out, attn_tensor *lse, void *stream);

/*
 * attn_sink_fwd that also returns the largest pre-softmax logit of every
 * (batch, query head): max over rows i and visible keys j of
 * scale * <q_i, k_j>, the sink excluded (page "Dao-AILab/flash-attention"
 * contributor guide, the task for issue #2986: users want the largest logit
 * before the softmax for monitoring, one value per batch and head, taken from
 * the row maxima the kernel computes anyway).
 *
 *   max_logit  [B, Hq] f32 (innermost stride 1), written completely: -inf
 *              where a (batch, head) has no position (L = 0).
 * Everything else as attn_sink_fwd.  The maxima come from the same fp32
 * scores the softmax uses.
 */
int attn_sink_fwd_max_logit(const attn_tensor *q, const attn_tensor *k, const attn_tensor *v,
                            const attn_tensor *sinks, int32_t window, float scale,
                            attn_tensor *out, attn_tensor *lse, attn_tensor *max_logit,
                            void *stream);

/*
 * Prefill forward over packed variable-length sequences (the varlen path of
 * page "Dao-AILab/flash-attention" contributor guide, call walk-through step
 * 2: cu_seqlens turned into per-sequence query tiles), with the learned sink
 * and window of attn_sink_fwd.  Each sequence is attended on its own: its
 * positions restart at 0 and no query sees another sequence's keys.
 *
 *   q           [T, Hq, D]  bf16, the sequences' rows one after another
 *   k, v        [T, Hkv, D] bf16
 *   cu_seqlens  [B + 1] int32, DEVICE memory: sequence b is rows
 *               cu_seqlens[b] .. cu_seqlens[b+1]-1; cu_seqlens[0] = 0,
 *               non-decreasing, cu_seqlens[B] = T (empty sequences allowed).
 *               Values are clamped to [0, T] on the device, so a malformed
 *               table gives wrong rows but no access outside the tensors.
 *   max_seqlen  host int >= every sequence's length (sizes the work grid;
 *               rows of a longer sequence past max_seqlen are not written).
 *   sinks, window, scale: as for attn_sink_fwd.
 *   out         [T, Hq, D]  bf16.
 *   lse         [Hq, T]     f32 or NULL (innermost stride 1).
 * Supported head dims D: 64, 128, 256.  B = 0, T = 0 or max_seqlen = 0 is a
 * no-op.  Runs on the tcgen05/TMEM tensor-core kernel of attn_sink_fwd.
 */
int attn_sink_fwd_varlen(const attn_tensor *q, const attn_tensor *k, const attn_tensor *v,
                         const attn_tensor *cu_seqlens, int32_t max_seqlen,
                         const attn_tensor *sinks, int32_t window, float scale,
                         attn_tensor *out, attn_tensor *lse, void *stream);

/*
 * The same operation on a plain CUDA-core fp32 kernel (one warp per output
 * row).  Slow; it is an independent second implementation for verification
 * and debugging, with the same arguments and semantics as attn_sink_fwd, and
 * any D that is a multiple of 32 up to 256.
 */
int attn_sink_fwd_cudacore(const attn_tensor *q, const attn_tensor *k,
                           const attn_tensor *v, const attn_tensor *sinks,
                           int32_t window, float scale, attn_tensor *out,
                           attn_tensor *lse, void *stream);

/*
 * Backward pass of attn_sink_fwd for the loss sum(dout * O): dq, dk, dv and
 * the sinks' gradient (page "Dao-AILab/flash-attention" contributor guide:
 * the FA4 backward's dK/dV and dQ phases, and issue #2969 on forming the
 * sink's gradient from the unrounded O).  With P_ij = exp(s_ij - LSE_i),
 * P_sink,i = exp(sink_h - LSE_i) and Dsum_i = dout_i . O_i:
 *   dv_j = sum_i P_ij dout_i;  dS_ij = P_ij (dout_i . v_j - Dsum_i);
 *   dq_i = scale sum_j dS_ij k_j;  dk_j = scale sum_i dS_ij q_i;
 *   dsink_h = -sum_{b,i} P_sink,i Dsum_i.
 *
 *   q, dout     [B, L, Hq, D]  bf16
 *   k, v        [B, L, Hkv, D] bf16
 *   o           [B, L, Hq, D]  the forward's output: bf16 (as attn_sink_fwd
 *               writes it; Dsum then carries its rounding) or f32 (Dsum exact,
 *               the form issue #2969 asks for); any outer strides (read with
 *               16-byte loads when they keep rows 16-byte aligned, else
 *               element by element)
 *   lse         [B, Hq, L]     f32, the forward's log-sum-exp (sink included)
 *   sinks, window, scale: as for attn_sink_fwd.
 *   dq          [B, L, Hq, D]  bf16, written completely
 *   dk, dv      [B, L, Hkv, D] bf16, written completely (summed over the
 *               query heads of each kv head)
 *   dsink       [Hq] f32, summed over the batch
 * D in {64, 128}.  Workspace, from the library's stream-ordered pool: fp32
 * dq accumulator and row sums, B*L*Hq*(D+1)*4 bytes, and fp32 dk and dv
 * accumulators, 2*B*L*Hkv*D*4 bytes.  The main pass runs on the
 * 5th-generation tensor cores (tcgen05, TMEM accumulators), accumulating in
 * fp32 with P and dS rounded to bf16 for the products.  Launches: a row
 * kernel (Dsum, the sink gradient, zeroed accumulators), the main pass, then
 * one fp32 -> bf16 conversion of dq, dk and dv; no host synchronisation.
 */
int attn_sink_bwd(const attn_tensor *q, const attn_tensor *k, const attn_tensor *v,
                  const attn_tensor *o, const attn_tensor *lse, const attn_tensor *dout,
                  const attn_tensor *sinks, int32_t window, float scale, attn_tensor *dq,
                  attn_tensor *dk, attn_tensor *dv, attn_tensor *dsink, void *stream);

/*
 * Single-token split-KV decode over a contiguous KV cache (page
 * "flashmla-optimization/docs/PATCH_STACK.md", section 3 "exact small-split
 * combine"; split-KV decode benchmark on the flash-attention contributor
 * guide page).
 *
 *   q        [B, Hq, D]       bf16; the query of sequence b sits at position
 *                             seqlens[b]-1 and its own key/value are already
 *                             in the cache.
 *   kcache,
 *   vcache   [B, Smax, Hkv, D] bf16; only positions < seqlens[b] are read.
 *   seqlens  [B] int32, DEVICE memory, 0 <= seqlens[b] <= Smax (values outside
 *            are clamped; a sequence of length 0 yields a zero output row).
 *   sinks    [Hq] f32, as for attn_sink_fwd.
 *   window   visible keys are [max(0, n-W), n-1] for n = seqlens[b].
 *   out      [B, Hq, D] bf16.
 *
 * Three launches on `stream`, no host synchronisation: a planner reads the
 * lengths on the device and splits each sequence's visible range into chunks;
 * a split kernel writes one partial (O_s, LSE_s) per (sequence, head, chunk);
 * a combine kernel merges only the chunks that exist, in chunk order, adding
 * the sink once.  The partials live in a workspace taken from a library-owned
 * stream-ordered memory pool (cudaMallocAsync/cudaFreeAsync on `stream`).
 * Supported: D in {64, 128, 256}, Hq/Hkv <= 16 (<= 8 at D = 256; larger groups
 * return ATTN_EUNSUPPORTED).
 */
int attn_sink_decode(const attn_tensor *q, const attn_tensor *kcache,
                     const attn_tensor *vcache, const attn_tensor *seqlens,
                     const attn_tensor *sinks, int32_t window, float scale,
                     attn_tensor *out, void *stream);

/*
 * attn_sink_decode with an explicit split size: `chunk` keys per split
 * (a positive multiple of 64, or 0 for the library's choice, which keeps every
 * sequence at <= 32 splits).  Used to force a given number of splits.
 */
int attn_sink_decode_chunked(const attn_tensor *q, const attn_tensor *kcache,
                             const attn_tensor *vcache, const attn_tensor *seqlens,
                             const attn_tensor *sinks, int32_t window, float scale,
                             int32_t chunk, attn_tensor *out, void *stream);

/*
 * Single-token split-KV decode over a PAGED KV cache (page
 * "Dao-AILab/flash-attention" contributor guide: module table row "Paged KV /
 * decode" and step 1 of its call walk-through, where the interface packs a
 * block_table; the window W of page "cf-1.com/news/6055759" applies as for
 * attn_sink_decode).
 *
 *   q            [B, Hq, D]        bf16, as for attn_sink_decode.
 *   kpages,
 *   vpages       [NB, P, Hkv, D]   bf16 pools of NB physical pages of P
 *                                  positions each; P a power of two in
 *                                  [16, 65536].
 *   block_table  [B, MP] int32, DEVICE memory (innermost stride 1): position
 *                t of sequence b is row t % P of page block_table[b][t / P].
 *                Pages may be shared between sequences.  An entry outside
 *                [0, NB) reads as a page of zero rows (no fault).  Entries of
 *                pages that hold no visible position may hold anything: they
 *                are either not read or read and discarded.
 *   seqlens      [B] int32, DEVICE memory, 0 <= n <= MP * P (clamped).
 *   sinks, window, scale, out: as for attn_sink_decode (Smax = MP * P).
 *
 * The same three launches as attn_sink_decode; each 64-key tile is loaded
 * from its page (P >= 64) or from 64/P pages (P = 16, 32) by TMA, so split
 * ranges start at the 64-key boundary at or below the window's first key and
 * the keys before the window are masked.  Workspace, supported D and Hq/Hkv:
 * as for attn_sink_decode.
 */
int attn_sink_decode_paged(const attn_tensor *q, const attn_tensor *kpages,
                           const attn_tensor *vpages, const attn_tensor *block_table,
                           const attn_tensor *seqlens, const attn_tensor *sinks,
                           int32_t window, float scale, attn_tensor *out, void *stream);

/*
 * Single-token split-KV decode over an FP8 (e4m3) KV cache, dequantised per kv
 * head (page "cf-1.com/news/6055759", "fix 2": the output scale is
 * rcp(row_sum) * sink_rescale * v_descale; its FP8 max_offset belongs to an
 * FP8 P, and P is not quantised here).
 *
 *   q          [B, Hq, D]        bf16, as for attn_sink_decode.
 *   kcache,
 *   vcache     [B, Smax, Hkv, D] ATTN_DTYPE_E4M3 bytes; every stride but the
 *                                innermost a multiple of 16 elements.
 *   k_descale,
 *   v_descale  [Hkv] f32, DEVICE memory: key row = k_descale[hk] * e4m3(row),
 *              value row likewise with v_descale.
 *   seqlens, sinks, window, scale, out: as for attn_sink_decode.
 *
 * The same three launches as attn_sink_decode; the split kernel streams the
 * e4m3 tiles (half the bytes of bf16), and each consumer warp converts its
 * keys and values to f16 in registers as it feeds them to the tensor cores
 * (exact: every e4m3 value is a normal f16 value); q enters in f16 under a
 * power-of-two scale, P in f16, and the key descale is folded into the
 * softmax scale, the value descale into the output scale.  D in {128, 256};
 * Hq/Hkv as for attn_sink_decode.
 */
int attn_sink_decode_fp8(const attn_tensor *q, const attn_tensor *kcache,
                         const attn_tensor *vcache, const attn_tensor *k_descale,
                         const attn_tensor *v_descale, const attn_tensor *seqlens,
                         const attn_tensor *sinks, int32_t window, float scale,
                         attn_tensor *out, void *stream);

/*
 * attn_sink_decode without any allocation (the pages have no counterpart to
 * this entry point; it is a deployment convenience).  Same arguments, result
 * and kernels as attn_sink_decode, but the split table and the partial
 * (O_s, LSE_s) live in a fixed 48 MiB array of device memory inside the
 * library instead of a stream-ordered allocation.  It is meant for callers
 * that may not allocate device memory while they decode: engines that
 * reserve nearly all of HBM for their KV cache up front and forbid library
 * allocations, or runtimes whose own allocator owns every device byte.
 *
 *  - Nothing is allocated or freed: no cudaMalloc/cudaFree of any kind.
 *  - The array is part of the library's device image: every GPU on which this
 *    entry point is used holds the 48 MiB until the process exits.
 *  - The first call on a device looks up the array's device address (with
 *    that device current); make that first call before any stream capture.
 *  - Workloads whose workspace bound exceeds 48 MiB are rejected with
 *    ATTN_EUNSUPPORTED and a message giving both sizes.  The bound is
 *    B * ceil(min(Smax, window) / chunk) * Hq * (D + 1) * 4 bytes, with the
 *    library's default chunk (every sequence <= 32 splits), plus ~1 KB.
 *  - All calls on a device share the one array and it keeps the last call's
 *    contents (each call rewrites everything it reads).  Calls whose kernels
 *    overlap on the GPU -- concurrent streams, or threads driving the same
 *    device -- race on it; serialise them (e.g. one stream).
 */
int attn_sink_decode_noalloc(const attn_tensor *q, const attn_tensor *kcache,
                             const attn_tensor *vcache, const attn_tensor *seqlens,
                             const attn_tensor *sinks, int32_t window, float scale,
                             attn_tensor *out, void *stream);

/*
 * Synchronises `stream`, then returns and clears the device status word of the
 * current device: ATTN_OK, ATTN_ETIMEOUT (a bounded wait ran out), or
 * ATTN_ECUDA if the synchronisation itself failed or a kernel found its launch
 * unusable (its dynamic shared memory not at the declared 1024-byte
 * alignment; it then returns before doing any work).
 */
int attn_sink_get_status(void *stream);

/*
 * Diagnostics: failure injection for tests of the error paths.  Not needed in
 * normal use (the pages have no counterpart to these).
 *
 * attn_sink_set_wait_limit_ns: the longest time any one device-side wait of
 * the kernels launched from now on may take on the current device before it
 * gives up, records ATTN_ETIMEOUT and lets its CTA return (0 restores the
 * default of 1 s).  With a limit of a few nanoseconds, the first wait that is
 * not satisfied at once gives up, so a call ends with ATTN_ETIMEOUT in the
 * status word and an unspecified output; the library stays usable.  Waits
 * that let a CTA's own copies land before it leaves keep the default limit.
 * Synchronous (a host-to-device copy); the setting is per device and shared
 * by every thread.
 *
 * attn_sink_fail_workspace_allocs: the next `count` workspace allocations
 * (decode, paged, FP8 and backward calls, any thread) fail as if the pool had
 * no memory: the call returns ATTN_ENOMEM and launches nothing.  0 cancels.
 */
int attn_sink_set_wait_limit_ns(uint64_t ns);
int attn_sink_fail_workspace_allocs(int32_t count);

/* Static description of an attn_status code. */
const char *attn_sink_strerror(int code);

/* One-line description of the last error returned on the calling thread
 * (empty string if none).  Valid until the next call on that thread. */
const char *attn_sink_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTNSINK_H */
