/*
 * oracle.c -- plain fp64 CPU oracle for sliding-window attention with one
 * learned sink logit per head.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file; it exists so that the CUDA kernels can be checked against
 * an obviously correct statement of what they compute.  It shares no code,
 * header, table or helper with the CUDA library.
 *
 * What is computed (page 1, "cf-1.com/news/6055759", section "why it must
 * change: Flint's learned sink"): each query attends to the W most recent keys
 * (itself included) and a per-head scalar "sink" logit joins the softmax
 * denominator as a virtual anchor that has no value row.  Page 1, "fix 2:
 * sink normalisation", fixes the numerics: the running maximum is taken over
 * the content logits AND the sink, so every exponent is <= 0, and the output
 * is scaled by the same factor as the denominator.  Here that is simply the
 * definition evaluated in double precision:
 *
 *   s_j  = scale * <q_i, k_j>                      j in V(i) = [max(0,i-W+1), i]
 *   M    = max(max_j s_j, sink)
 *   Z    = sum_j exp(s_j - M) + exp(sink - M)
 *   O_i  = sum_j exp(s_j - M) v_j / Z
 *   LSE_i = M + ln Z                                (natural log, sink included)
 *
 * Readings taken where the pages are silent (each one is listed in the design
 * notes): the sink is a logit in post-scale units and is not multiplied by
 * `scale` (page 1, fix 2 multiplies only sink_val by log2(e) but row_max by the
 * scaled log2 factor); query head h reads kv head h / (Hq/Hkv); the FP8-only
 * max_offset and v_descale terms of page 1 are 0 and 1 for bf16 inputs.
 *
 * Split-KV decode (page 5, "PATCH_STACK.md", section 3 "exact small-split
 * combine") is stated here as its two steps: a partial softmax over one key
 * range (no sink) producing (O_s, LSE_s), and the log-sum-exp merge of the
 * splits that exist, in split order, with the sink added once.
 *
 * Inputs are bf16 bit patterns (uint16) so that the oracle reads exactly the
 * bits the device reads; each is widened exactly to double.  Sinks and scale
 * arrive as float32 and are widened exactly.  OpenMP parallelises over rows.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_to_f64(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * One output row: query vector q (D bf16), keys/values are the rows
 * k[j*kstride .. +D), v[j*vstride .. +D) for j in [lo, hi] (inclusive).
 * sink may be -INFINITY.  Writes D outputs and the natural-log LSE.
 * s is caller-provided scratch of at least hi-lo+1 doubles.
 */
static void attend_row(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                       int64_t kvstride, int lo, int hi, int D, double scale,
                       double sink, double *s, double *out, double *lse)
{
    int n = hi - lo + 1;
    double M = sink;
    for (int t = 0; t < n; ++t) {
        const uint16_t *kr = k + (int64_t)(lo + t) * kvstride;
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
            dot += bf16_to_f64(q[d]) * bf16_to_f64(kr[d]);
        s[t] = scale * dot;
        if (s[t] > M) M = s[t];
    }
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    if (n <= 0 && isinf(sink) && sink < 0) {
        /* No content key and no sink: the softmax is empty.  Never reached
         * through the public paths (the diagonal key is always visible and a
         * zero-length decode sequence is reported separately). */
        *lse = -INFINITY;
        return;
    }
    double Z = (isinf(sink) && sink < 0) ? 0.0 : exp(sink - M);
    for (int t = 0; t < n; ++t) {
        double p = exp(s[t] - M);
        Z += p;
        const uint16_t *vr = v + (int64_t)(lo + t) * kvstride;
        for (int d = 0; d < D; ++d) out[d] += p * bf16_to_f64(vr[d]);
    }
    for (int d = 0; d < D; ++d) out[d] /= Z;
    *lse = M + log(Z);
}

/*
 * Prefill forward.  q [B,L,Hq,D], k/v [B,L,Hkv,D] bf16 bits, sinks [Hq] f32.
 * out [B,L,Hq,D] f64, lse [B,Hq,L] f64 (lse may be NULL).
 * Returns 0, or -1 on invalid sizes.
 */
int oracle_fwd(const uint16_t *q, const uint16_t *k, const uint16_t *v,
               const float *sinks, int B, int L, int Hq, int Hkv, int D,
               int W, float scale, double *out, double *lse)
{
    if (B < 0 || L < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || W < 1 || Hq % Hkv)
        return -1;
    const int group = Hq / Hkv;
    const int64_t rows = (int64_t)B * L * Hq;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
        double lse_row;
#pragma omp for schedule(dynamic, 64)
        for (int64_t r = 0; r < rows; ++r) {
            int h = (int)(r % Hq);
            int i = (int)((r / Hq) % L);
            int b = (int)(r / ((int64_t)Hq * L));
            int hk = h / group;
            int lo = i - W + 1 < 0 ? 0 : i - W + 1;
            const uint16_t *qr = q + (((int64_t)b * L + i) * Hq + h) * D;
            const uint16_t *kb = k + ((int64_t)b * L * Hkv + hk) * D;
            const uint16_t *vb = v + ((int64_t)b * L * Hkv + hk) * D;
            attend_row(qr, kb, vb, (int64_t)Hkv * D, lo, i, D, (double)scale,
                       (double)sinks[h], s,
                       out + (((int64_t)b * L + i) * Hq + h) * D, &lse_row);
            if (lse) lse[((int64_t)b * Hq + h) * L + i] = lse_row;
        }
        free(s);
    }
    return 0;
}

/*
 * The same forward, for a chosen list of rows only (for sizes where the whole
 * output would take too long).  rows: nrows triples (b, i, h).
 * out [nrows, D], lse [nrows].
 */
int oracle_fwd_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                    const float *sinks, int B, int L, int Hq, int Hkv, int D,
                    int W, float scale, int nrows, const int32_t *rows,
                    double *out, double *lse)
{
    if (B < 0 || L < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || W < 1 || Hq % Hkv)
        return -1;
    for (int r = 0; r < nrows; ++r) {
        int b = rows[3 * r], i = rows[3 * r + 1], h = rows[3 * r + 2];
        if (b < 0 || b >= B || i < 0 || i >= L || h < 0 || h >= Hq) return -1;
    }
    const int group = Hq / Hkv;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
#pragma omp for schedule(dynamic, 1)
        for (int r = 0; r < nrows; ++r) {
            int b = rows[3 * r], i = rows[3 * r + 1], h = rows[3 * r + 2];
            int hk = h / group;
            int lo = i - W + 1 < 0 ? 0 : i - W + 1;
            const uint16_t *qr = q + (((int64_t)b * L + i) * Hq + h) * D;
            const uint16_t *kb = k + ((int64_t)b * L * Hkv + hk) * D;
            const uint16_t *vb = v + ((int64_t)b * L * Hkv + hk) * D;
            attend_row(qr, kb, vb, (int64_t)Hkv * D, lo, i, D, (double)scale,
                       (double)sinks[h], s, out + (int64_t)r * D, lse + r);
        }
        free(s);
    }
    return 0;
}

/*
 * Single-token decode over a contiguous KV cache.  q [B,Hq,D],
 * kcache/vcache [B,Smax,Hkv,D] bf16 bits, seqlens [B] int32 (0..Smax).
 * The query sits at position n-1 of its sequence and sees the keys
 * [max(0, n-W), n-1].  A sequence with n == 0 has only the sink in its
 * softmax, so its output row is 0 and its LSE is the sink.
 * out [B,Hq,D] f64, lse [B,Hq] f64 (may be NULL).
 */
int oracle_decode(const uint16_t *q, const uint16_t *kc, const uint16_t *vc,
                  const int32_t *seqlens, const float *sinks, int B, int Smax,
                  int Hq, int Hkv, int D, int W, float scale, double *out,
                  double *lse)
{
    if (B < 0 || Smax < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || W < 1 || Hq % Hkv)
        return -1;
    for (int b = 0; b < B; ++b)
        if (seqlens[b] < 0 || seqlens[b] > Smax) return -1;
    const int group = Hq / Hkv;
    const int64_t rows = (int64_t)B * Hq;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Smax > 0 ? Smax : 1));
        double lse_row;
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < rows; ++r) {
            int h = (int)(r % Hq);
            int b = (int)(r / Hq);
            int hk = h / group;
            int n = seqlens[b];
            int lo = n - W < 0 ? 0 : n - W;
            const uint16_t *kb = kc + ((int64_t)b * Smax * Hkv + hk) * D;
            const uint16_t *vb = vc + ((int64_t)b * Smax * Hkv + hk) * D;
            attend_row(q + r * D, kb, vb, (int64_t)Hkv * D, lo, n - 1, D,
                       (double)scale, (double)sinks[h], s, out + r * D, &lse_row);
            if (lse) lse[r] = lse_row;
        }
        free(s);
    }
    return 0;
}

/*
 * Single-token decode over a paged KV cache (page 4, "Dao-AILab/flash-attention"
 * contributor guide: the module table's "Paged KV / decode" row and step 1 of
 * its call walk-through, where the interface packs a block_table; page 1's
 * sliding-window serving with W = 513).  The cache is a pool of NB physical
 * pages of P positions, kp/vp [NB, P, Hkv, D] bf16 bits, and block_table
 * [B, MP] int32 maps page number t / P of sequence b to its physical page:
 * position t of sequence b is row t % P of page block_table[b * MP + t / P].
 * An entry outside [0, NB) stands for a page whose rows are all zero.  With
 * that cache, the result is oracle_decode's with Smax = MP * P: the query at
 * position n-1 sees the keys [max(0, n-W), n-1] and the sink.
 * out [B,Hq,D] f64, lse [B,Hq] f64 (may be NULL).
 */
int oracle_decode_paged(const uint16_t *q, const uint16_t *kp, const uint16_t *vp,
                        const int32_t *block_table, const int32_t *seqlens,
                        const float *sinks, int B, int NB, int P, int MP, int Hq,
                        int Hkv, int D, int W, float scale, double *out,
                        double *lse)
{
    if (B < 0 || NB < 0 || P <= 0 || MP < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 ||
        W < 1 || Hq % Hkv)
        return -1;
    const int64_t smax = (int64_t)MP * P;
    for (int b = 0; b < B; ++b)
        if (seqlens[b] < 0 || seqlens[b] > smax) return -1;
    const int group = Hq / Hkv;
    const int64_t rows = (int64_t)B * Hq;
#pragma omp parallel
    {
        /* the visible rows of one (sequence, kv head), gathered in order */
        uint16_t *kr = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(smax > 0 ? smax : 1) * D);
        uint16_t *vr = (uint16_t *)malloc(sizeof(uint16_t) * (size_t)(smax > 0 ? smax : 1) * D);
        double *s = (double *)malloc(sizeof(double) * (size_t)(smax > 0 ? smax : 1));
        double lse_row;
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < rows; ++r) {
            int h = (int)(r % Hq);
            int b = (int)(r / Hq);
            int hk = h / group;
            int n = seqlens[b];
            int lo = n - W < 0 ? 0 : n - W;
            for (int t = lo; t < n; ++t) {
                int32_t page = block_table[(int64_t)b * MP + t / P];
                int slot = t % P;
                uint16_t *kd = kr + (int64_t)(t - lo) * D;
                uint16_t *vd = vr + (int64_t)(t - lo) * D;
                if (page < 0 || page >= NB) {
                    memset(kd, 0, sizeof(uint16_t) * (size_t)D);
                    memset(vd, 0, sizeof(uint16_t) * (size_t)D);
                } else {
                    int64_t off = (((int64_t)page * P + slot) * Hkv + hk) * D;
                    memcpy(kd, kp + off, sizeof(uint16_t) * (size_t)D);
                    memcpy(vd, vp + off, sizeof(uint16_t) * (size_t)D);
                }
            }
            attend_row(q + r * D, kr, vr, D, 0, n - lo - 1, D, (double)scale,
                       (double)sinks[h], s, out + r * D, &lse_row);
            if (lse) lse[r] = lse_row;
        }
        free(s);
        free(vr);
        free(kr);
    }
    return 0;
}

/*
 * FP8 e4m3 (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent
 * 0 is subnormal, m * 2^-9; S.1111.111 is NaN; no infinities) to double,
 * written from that definition.
 */
static double e4m3_to_f64(uint8_t b)
{
    int sign = b >> 7, e = (b >> 3) & 15, m = b & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -v : v;
}

double oracle_e4m3_to_f64(uint8_t b) { return e4m3_to_f64(b); }

/*
 * Single-token decode over an FP8 (e4m3) KV cache with one dequantisation
 * scale per kv head: the key row is k_descale[hk] * e4m3(kc row) and the value
 * row v_descale[hk] * e4m3(vc row).  Page 1, "fix 2", applies v_descale to the
 * output scale (rcp(row_sum) * sink_rescale * v_descale); its FP8 max_offset
 * belongs to an FP8 P, and P is not quantised here, so it is 0.  Otherwise as
 * oracle_decode: kc/vc [B,Smax,Hkv,D] bytes, out [B,Hq,D], lse [B,Hq].
 */
int oracle_decode_fp8(const uint16_t *q, const uint8_t *kc, const uint8_t *vc,
                      const float *k_descale, const float *v_descale,
                      const int32_t *seqlens, const float *sinks, int B, int Smax,
                      int Hq, int Hkv, int D, int W, float scale, double *out,
                      double *lse)
{
    if (B < 0 || Smax < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || W < 1 || Hq % Hkv)
        return -1;
    for (int b = 0; b < B; ++b)
        if (seqlens[b] < 0 || seqlens[b] > Smax) return -1;
    const int group = Hq / Hkv;
    const int64_t rows = (int64_t)B * Hq;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(Smax > 0 ? Smax : 1));
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < rows; ++r) {
            int h = (int)(r % Hq);
            int b = (int)(r / Hq);
            int hk = h / group;
            int n = seqlens[b];
            int lo = n - W < 0 ? 0 : n - W;
            double ks = (double)k_descale[hk], vs = (double)v_descale[hk];
            const uint16_t *qr = q + r * D;
            double M = (double)sinks[h];
            for (int t = lo; t < n; ++t) {
                const uint8_t *kr = kc + (((int64_t)b * Smax + t) * Hkv + hk) * D;
                double dot = 0.0;
                for (int d = 0; d < D; ++d)
                    dot += bf16_to_f64(qr[d]) * (ks * e4m3_to_f64(kr[d]));
                s[t - lo] = (double)scale * dot;
                if (s[t - lo] > M) M = s[t - lo];
            }
            double *o = out + r * D;
            for (int d = 0; d < D; ++d) o[d] = 0.0;
            double Z = (isinf((double)sinks[h]) && sinks[h] < 0) ? 0.0 : exp((double)sinks[h] - M);
            for (int t = lo; t < n; ++t) {
                double p = exp(s[t - lo] - M);
                Z += p;
                const uint8_t *vr = vc + (((int64_t)b * Smax + t) * Hkv + hk) * D;
                for (int d = 0; d < D; ++d) o[d] += p * (vs * e4m3_to_f64(vr[d]));
            }
            if (Z > 0.0) {
                for (int d = 0; d < D; ++d) o[d] /= Z;
                if (lse) lse[r] = M + log(Z);
            } else if (lse) {
                lse[r] = -INFINITY;
            }
        }
        free(s);
    }
    return 0;
}

/*
 * Split-KV step 1 (page 5, section 3): the partial softmax of one query row
 * over the keys [lo, hi] only, with no sink.  O_s is normalised within the
 * split and LSE_s is its natural-log normaliser.  Requires lo <= hi.
 * q [D], k/v rows at stride kvstride elements.
 */
int oracle_split_partial(const uint16_t *q, const uint16_t *k,
                         const uint16_t *v, int64_t kvstride, int lo, int hi,
                         int D, float scale, double *o_s, double *lse_s)
{
    if (lo < 0 || hi < lo || D <= 0) return -1;
    double *s = (double *)malloc(sizeof(double) * (size_t)(hi - lo + 1));
    attend_row(q, k, v, kvstride, lo, hi, D, (double)scale, -INFINITY, s, o_s,
               lse_s);
    free(s);
    return 0;
}

/*
 * Split-KV step 2 (page 5, section 3): merge the nsplits partials that exist,
 * in split order 0, 1, ..., with the sink joining the denominator once.
 *   M   = max(max_s LSE_s, sink)
 *   w_s = exp(LSE_s - M),  w_sink = exp(sink - M),  Den = sum_s w_s + w_sink
 *   O   = sum_s w_s O_s / Den,   LSE = M + ln Den
 * With nsplits == 0 the output is 0 and LSE is the sink.
 */
int oracle_combine(int nsplits, const double *lse_s, const double *o_s, int D,
                   float sink, double *out, double *lse)
{
    if (nsplits < 0 || D <= 0) return -1;
    double M = (double)sink;
    for (int s = 0; s < nsplits; ++s)
        if (lse_s[s] > M) M = lse_s[s];
    double den = (isinf((double)sink) && sink < 0) ? 0.0 : exp((double)sink - M);
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    for (int s = 0; s < nsplits; ++s) {
        double w = exp(lse_s[s] - M);
        den += w;
        for (int d = 0; d < D; ++d) out[d] += w * o_s[(int64_t)s * D + d];
    }
    if (den > 0.0) {
        for (int d = 0; d < D; ++d) out[d] /= den;
        *lse = M + log(den);
    } else {
        *lse = -INFINITY;
    }
    return 0;
}
