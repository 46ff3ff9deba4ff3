"""Pins for the fp64 oracle: each test checks it against something other than
itself -- a library routine, a closed form, an invariant or a brute-force
formulation -- so that a dropped term, a wrong sign or index, or a transposed
operand anywhere in it fails at least one test.  CPU only."""
import math

import numpy as np
import pytest
import scipy.special as sps
import torch

import oracle
from sliding_window_learned_b200 import inputs


def _rand_case(rng, B, L, Hq, Hkv, D, sink_lo=-4.0, sink_hi=8.0, scale=None):
    q = torch.from_numpy(rng.standard_normal((B, L, Hq, D)).astype(np.float32)).bfloat16()
    k = torch.from_numpy(rng.standard_normal((B, L, Hkv, D)).astype(np.float32)).bfloat16()
    v = torch.from_numpy(rng.standard_normal((B, L, Hkv, D)).astype(np.float32)).bfloat16()
    sinks = rng.uniform(sink_lo, sink_hi, Hq).astype(np.float32)
    if scale is None:
        scale = float(np.float32(1.0 / math.sqrt(D)))
    return q, k, v, sinks, scale


def _f64(t):
    return t.double().numpy()


def _scores(q, k, Hq, Hkv, scale):
    """Plain scores via a library matmul: [B, Hq, L, L] in float64."""
    qd = torch.from_numpy(_f64(q)).permute(0, 2, 1, 3)           # B Hq L D
    kd = torch.from_numpy(_f64(k)).permute(0, 2, 1, 3)           # B Hkv L D
    kd = kd.repeat_interleave(Hq // Hkv, dim=1)                  # B Hq L D
    return (torch.matmul(qd, kd.transpose(-1, -2)) * scale).numpy()


def _window_mask(L, W):
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    return (j <= i) & (j >= i - W + 1)


# ---------------------------------------------------------------- brute force
@pytest.mark.parametrize("D", [4, 64])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 2)])
@pytest.mark.parametrize("L", [1, 5, 16])
def test_brute_force_dense_sink_column(D, Hq, Hkv, L):
    """Independent dense formulation: an (L+1)-wide softmax matrix whose extra
    column holds the sink logit and has no value row (page 1, learned sink as a
    virtual anchor logit in the denominator).  Every W in 1..L+1."""
    rng = np.random.default_rng(1000 * D + 10 * L + Hq)
    B = 2
    q, k, v, sinks, scale = _rand_case(rng, B, L, Hq, Hkv, D)
    S = _scores(q, k, Hq, Hkv, scale)                            # B Hq L L
    vd = np.repeat(_f64(v).transpose(0, 2, 1, 3), Hq // Hkv, axis=1)  # B Hq L D
    for W in range(1, L + 2):
        mask = _window_mask(L, W)
        big = np.full((B, Hq, L, L + 1), -np.inf)
        big[..., 0] = sinks[None, :, None]
        big[..., 1:] = np.where(mask, S, -np.inf)
        P = sps.softmax(big, axis=-1)
        O_ref = np.einsum("bhij,bhjd->bihd", P[..., 1:], vd)
        lse_ref = sps.logsumexp(big, axis=-1)
        O, lse = oracle.fwd(inputs.bits(q), inputs.bits(k), inputs.bits(v), sinks, W, scale)
        np.testing.assert_allclose(O, O_ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, lse_ref, rtol=1e-13, atol=1e-12)


# ------------------------------------------------- sink -> -inf == library SDPA
@pytest.mark.parametrize("L,W,Hq,Hkv,D", [(37, 5, 4, 2, 16), (64, 64, 2, 1, 32), (50, 1, 3, 3, 8),
                                          (70, 33, 8, 2, 64)])
def test_sink_minus_inf_is_plain_window_attention(L, W, Hq, Hkv, D):
    """With sink = -inf the method is plain causal sliding-window softmax
    attention: compare with torch's scaled_dot_product_attention in float64
    (a library routine) and its LSE with torch.logsumexp."""
    rng = np.random.default_rng(L * W + D)
    q, k, v, _, scale = _rand_case(rng, 2, L, Hq, Hkv, D)
    sinks = np.full(Hq, -np.inf, np.float32)
    O, lse = oracle.fwd(inputs.bits(q), inputs.bits(k), inputs.bits(v), sinks, W, scale)
    qd = q.double().permute(0, 2, 1, 3)
    kd = k.double().permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, 1)
    vd = v.double().permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, 1)
    mask = torch.from_numpy(_window_mask(L, W))
    ref = torch.nn.functional.scaled_dot_product_attention(qd, kd, vd, attn_mask=mask, scale=scale)
    np.testing.assert_allclose(O, ref.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)
    s = torch.matmul(qd, kd.transpose(-1, -2)) * scale
    lse_ref = torch.logsumexp(s.masked_fill(~mask, float("-inf")), dim=-1)
    np.testing.assert_allclose(lse, lse_ref.numpy(), rtol=1e-13, atol=1e-12)


# ------------------------------------------- finite sink: closed form from SDPA
@pytest.mark.parametrize("sink_lo,sink_hi", [(-4, 8), (-60, -40), (15, 25)])
def test_finite_sink_closed_form(sink_lo, sink_hi):
    """A finite sink rescales plain attention:  O_sink = O_plain * sigmoid(LSE_plain - sink)
    and LSE_sink = logaddexp(LSE_plain, sink), with O_plain/LSE_plain from the
    library routines.  Pins the sink term (no scale on the sink, added once)."""
    L, W, Hq, Hkv, D = 45, 17, 4, 2, 32
    rng = np.random.default_rng(sink_hi + 100)
    q, k, v, sinks, scale = _rand_case(rng, 2, L, Hq, Hkv, D, sink_lo, sink_hi)
    O, lse = oracle.fwd(inputs.bits(q), inputs.bits(k), inputs.bits(v), sinks, W, scale)
    qd = q.double().permute(0, 2, 1, 3)
    kd = k.double().permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, 1)
    vd = v.double().permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, 1)
    mask = torch.from_numpy(_window_mask(L, W))
    Op = torch.nn.functional.scaled_dot_product_attention(qd, kd, vd, attn_mask=mask, scale=scale)
    s = torch.matmul(qd, kd.transpose(-1, -2)) * scale
    lp = torch.logsumexp(s.masked_fill(~mask, float("-inf")), dim=-1)       # B Hq L
    sk = torch.from_numpy(sinks.astype(np.float64))[None, :, None]
    fac = torch.sigmoid(lp - sk)                                           # B Hq L
    O_ref = (Op * fac[..., None]).permute(0, 2, 1, 3).numpy()
    lse_ref = torch.logaddexp(lp, sk.expand_as(lp)).numpy()
    np.testing.assert_allclose(O, O_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-13, atol=1e-11)


# ------------------------------------------------------------- special windows
def test_window_at_least_L_is_full_causal():
    """W >= L gives exactly full causal attention (bit-identical in the oracle),
    and equals SDPA's is_causal with sink = -inf."""
    L, Hq, Hkv, D = 40, 4, 1, 16
    rng = np.random.default_rng(7)
    q, k, v, sinks, scale = _rand_case(rng, 1, L, Hq, Hkv, D)
    args = (inputs.bits(q), inputs.bits(k), inputs.bits(v))
    O1, l1 = oracle.fwd(*args, sinks, L, scale)
    for W in (L + 1, 3 * L, 2**31 - 1):
        O2, l2 = oracle.fwd(*args, sinks, W, scale)
        assert np.array_equal(O1, O2) and np.array_equal(l1, l2)
    ninf = np.full(Hq, -np.inf, np.float32)
    O3, _ = oracle.fwd(*args, ninf, L, scale)
    qd = q.double().permute(0, 2, 1, 3)
    kd = k.double().permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, 1)
    vd = v.double().permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, 1)
    ref = torch.nn.functional.scaled_dot_product_attention(qd, kd, vd, is_causal=True, scale=scale)
    np.testing.assert_allclose(O3, ref.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)


def test_window_one_closed_form():
    """W = 1: O_i = V_i e^{s_ii} / (e^{s_ii} + e^{sink}), LSE_i = logaddexp(s_ii, sink)."""
    L, Hq, Hkv, D = 33, 4, 2, 64
    rng = np.random.default_rng(11)
    q, k, v, sinks, scale = _rand_case(rng, 2, L, Hq, Hkv, D)
    O, lse = oracle.fwd(inputs.bits(q), inputs.bits(k), inputs.bits(v), sinks, 1, scale)
    qd, kd, vd = _f64(q), _f64(k), _f64(v)
    g = Hq // Hkv
    for b in range(2):
        for h in range(Hq):
            sii = scale * np.einsum("id,id->i", qd[b, :, h], kd[b, :, h // g])
            w = sps.expit(sii - sinks[h])
            np.testing.assert_allclose(O[b, :, h], vd[b, :, h // g] * w[:, None], rtol=0, atol=1e-13)
            np.testing.assert_allclose(lse[:, h][b], np.logaddexp(sii, sinks[h]), rtol=1e-14, atol=1e-13)


def test_sink_far_above_content_drives_output_to_zero():
    """The stress construction (content logits near -150) with sinks +20/-50:
    ||O_i||_inf <= e^{max s - sink} max|v| and LSE -> sink for the +20 heads;
    everything finite."""
    cfg = inputs.Prefill("stress-small", 1, 96, 4, 2, 256, 33, ("split", 20.0, -50.0),
                         qk_offset=inputs.STRESS.qk_offset)
    x = inputs.make_prefill(cfg, seed=3)
    O, lse = oracle.fwd(inputs.bits(x["q"]), inputs.bits(x["k"]), inputs.bits(x["v"]),
                        x["sinks"].numpy(), cfg.W, cfg.scale)
    assert np.isfinite(O).all() and np.isfinite(lse).all()
    S = _scores(x["q"], x["k"], cfg.Hq, cfg.Hkv, cfg.scale)[0]          # Hq L L
    mask = _window_mask(cfg.L, cfg.W)
    smax = np.where(mask, S, -np.inf).max(-1)                           # Hq L
    assert (smax < -100).all() and (np.where(mask, S, 0).min() > -200)
    vmax = np.abs(_f64(x["v"])).max()
    for h in range(cfg.Hq):
        sink = float(x["sinks"][h])
        bound = np.exp(smax[h] - sink) * vmax * cfg.W
        assert (np.abs(O[0, :, h]).max(-1) <= bound + 1e-300).all()
        if sink > 0:
            np.testing.assert_allclose(lse[0, h], sink, rtol=0, atol=1e-40)


# ----------------------------------------------------------------- invariants
def test_probability_mass_bound():
    """Content weights and the sink weight sum to one, so
    |O_i|_inf <= (1 - P_sink,i) max_j |v_j|_inf with P_sink = e^{sink - LSE}."""
    L, W, Hq, Hkv, D = 80, 20, 4, 2, 32
    rng = np.random.default_rng(5)
    q, k, v, sinks, scale = _rand_case(rng, 1, L, Hq, Hkv, D)
    O, lse = oracle.fwd(inputs.bits(q), inputs.bits(k), inputs.bits(v), sinks, W, scale)
    vmax = np.abs(_f64(v)).max()
    p_sink = np.exp(sinks[None, :, None] - lse)                        # B Hq L
    bound = (1 - p_sink) * vmax
    assert (np.abs(O).max(-1) <= bound.transpose(0, 2, 1) + 1e-12).all()
    assert ((p_sink > 0) & (p_sink < 1)).all()


def test_shift_invariance_with_sink():
    """Adding the same constant to every content logit and to the sink leaves O
    unchanged and shifts LSE by the constant.  The constant enters through an
    extra head dimension (q_D = 1, k_D = 8, scale = 1/8: +1 on every logit)."""
    L, W, Hq, Hkv, D = 30, 7, 2, 1, 15
    rng = np.random.default_rng(9)
    q, k, v, sinks, _ = _rand_case(rng, 1, L, Hq, Hkv, D)
    scale = 0.125
    q1 = torch.cat([q, torch.zeros(1, L, Hq, 1, dtype=torch.bfloat16)], -1)
    k1 = torch.cat([k, torch.zeros(1, L, Hkv, 1, dtype=torch.bfloat16)], -1)
    v1 = torch.cat([v, torch.zeros(1, L, Hkv, 1, dtype=torch.bfloat16)], -1)
    q2 = torch.cat([q, torch.ones(1, L, Hq, 1, dtype=torch.bfloat16)], -1)
    k2 = torch.cat([k, torch.full((1, L, Hkv, 1), 8.0, dtype=torch.bfloat16)], -1)
    O1, l1 = oracle.fwd(inputs.bits(q1), inputs.bits(k1), inputs.bits(v1), sinks, W, scale)
    O2, l2 = oracle.fwd(inputs.bits(q2), inputs.bits(k2), inputs.bits(v1), sinks + 1.0, W, scale)
    np.testing.assert_allclose(O2, O1, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l2, l1 + 1.0, rtol=0, atol=1e-12)


def test_rows_entry_matches_full():
    L, W, Hq, Hkv, D = 50, 9, 4, 2, 16
    rng = np.random.default_rng(12)
    q, k, v, sinks, scale = _rand_case(rng, 2, L, Hq, Hkv, D)
    a = (inputs.bits(q), inputs.bits(k), inputs.bits(v), sinks, W, scale)
    O, lse = oracle.fwd(*a)
    rows = np.array([[0, 0, 0], [1, 49, 3], [0, 17, 2], [1, 8, 1]])
    Or, lr = oracle.fwd_rows(*a, rows)
    for n, (b, i, h) in enumerate(rows):
        assert np.array_equal(Or[n], O[b, i, h]) and lr[n] == lse[b, h, i]


# --------------------------------------------------------------------- decode
def test_decode_matches_dense_last_row():
    """Decode at length n is the forward's row n-1 over the cached keys,
    checked against the dense sink-column softmax; poisoned slots past n are
    never read; n = 0 gives O = 0 and LSE = sink."""
    rng = np.random.default_rng(21)
    B, Smax, Hq, Hkv, D = 5, 40, 8, 2, 16
    seqlens = np.array([1, 17, 40, 0, 33], np.int32)
    for W in (1, 6, 40, 1000):
        q = torch.from_numpy(rng.standard_normal((B, Hq, D)).astype(np.float32)).bfloat16()
        kc = torch.from_numpy(rng.standard_normal((B, Smax, Hkv, D)).astype(np.float32)).bfloat16()
        vc = torch.from_numpy(rng.standard_normal((B, Smax, Hkv, D)).astype(np.float32)).bfloat16()
        for b in range(B):
            kc[b, seqlens[b]:] = float("nan")
            vc[b, seqlens[b]:] = float("nan")
        sinks = rng.uniform(-4, 8, Hq).astype(np.float32)
        scale = 0.25
        O, lse = oracle.decode(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), seqlens, sinks, W, scale)
        for b in range(B):
            n = int(seqlens[b])
            lo = max(0, n - W)
            for h in range(Hq):
                hk = h // (Hq // Hkv)
                s = scale * (_f64(kc[b, lo:n, hk]) @ _f64(q[b, h]))
                row = np.concatenate([[sinks[h]], s])
                p = sps.softmax(row)
                ref = p[1:] @ _f64(vc[b, lo:n, hk]) if n else np.zeros(D)
                np.testing.assert_allclose(O[b, h], ref, rtol=0, atol=1e-12)
                np.testing.assert_allclose(lse[b, h], sps.logsumexp(row), rtol=1e-14, atol=1e-12)


@pytest.mark.parametrize("nsplits", [1, 2, 31, 32, 33, "uneven"])
def test_split_combine_is_exact(nsplits):
    """Page 5, section 3: merging the partial (O_s, LSE_s) of any partition of
    the keys, over the splits that exist only, equals the unsplit result."""
    rng = np.random.default_rng(31)
    n, Hq, D = 300, 4, 32
    q = torch.from_numpy(rng.standard_normal((1, Hq, D)).astype(np.float32)).bfloat16()
    kc = torch.from_numpy(rng.standard_normal((1, n, 1, D)).astype(np.float32)).bfloat16()
    vc = torch.from_numpy(rng.standard_normal((1, n, 1, D)).astype(np.float32)).bfloat16()
    sinks = np.array([-np.inf, -3.0, 2.0, 30.0], np.float32)
    scale = 0.2
    O, lse = oracle.decode(inputs.bits(q), inputs.bits(kc), inputs.bits(vc),
                           np.array([n], np.int32), sinks, n, scale)
    if nsplits == "uneven":
        cuts = [0, 1, 2, 50, 51, 180, 299, 300]
    else:
        cuts = [round(i * n / nsplits) for i in range(nsplits + 1)]
    kb, vb = inputs.bits(kc[0, :, 0]), inputs.bits(vc[0, :, 0])
    for h in range(Hq):
        parts = [oracle.split_partial(inputs.bits(q[0, h]), kb, vb, a, b - 1, scale)
                 for a, b in zip(cuts[:-1], cuts[1:]) if b > a]
        o_s = np.stack([p[0] for p in parts])
        l_s = np.array([p[1] for p in parts])
        Oc, lc = oracle.combine(l_s, o_s, sinks[h])
        np.testing.assert_allclose(Oc, O[0, h], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lc, lse[0, h], rtol=1e-14, atol=1e-12)


def test_combine_with_no_splits_is_sink_only():
    out, lse = oracle.combine(np.zeros(0), np.zeros((0, 8)), 1.5)
    assert np.array_equal(out, np.zeros(8)) and lse == 1.5


# -------------------------------------------- the overflow the rebasing removes
def test_old_sink_term_overflows_and_rebased_one_does_not():
    """Page 1, fix 2.  Re-enact the running-softmax sink update in float32 on
    the stress construction: adding exp2(sink*log2e - row_max*scale_log2) to
    the row sum overflows float32 when the sink sits ~170 above the content
    maximum (output 0 or NaN), while rebasing the maximum on the sink stays
    finite and agrees with the oracle."""
    cfg = inputs.Prefill("stress-small", 1, 64, 2, 1, 256, 64, ("split", 20.0, -50.0),
                         qk_offset=inputs.STRESS.qk_offset)
    x = inputs.make_prefill(cfg, seed=4)
    O, _ = oracle.fwd(inputs.bits(x["q"]), inputs.bits(x["k"]), inputs.bits(x["v"]),
                      x["sinks"].numpy(), cfg.W, cfg.scale)
    f = np.float32
    log2e = f(1.4426950408889634)
    S = _scores(x["q"], x["k"], cfg.Hq, cfg.Hkv, 1.0)[0].astype(np.float32)  # raw QK^T
    vv = x["v"].float().numpy()[0, :, 0]
    scale_log2 = f(cfg.scale) * log2e
    i = cfg.L - 1
    h = 0                                                               # sink = +20
    sink = f(x["sinks"][h])
    s = S[h, i, : i + 1]
    row_max = s.max()
    p = np.exp2(s * scale_log2 - row_max * scale_log2).astype(np.float32)
    acc = (p[:, None] * vv[: i + 1]).sum(0, dtype=np.float32)
    row_sum = p.sum(dtype=np.float32)
    with np.errstate(over="ignore", invalid="ignore"):
        old_sum = row_sum + np.exp2(f(sink * log2e - row_max * scale_log2))
        old_out = acc * (f(1) / old_sum)
    assert not np.isfinite(old_sum) and (np.all(old_out == 0) or np.isnan(old_out).any())
    old_l2 = row_max * scale_log2
    new_l2 = max(old_l2, sink * log2e)
    r = np.exp2(f(old_l2 - new_l2))
    new_sum = row_sum * r + np.exp2(f(sink * log2e - new_l2))
    new_out = acc * (f(1) / new_sum) * r
    assert np.isfinite(new_out).all()
    np.testing.assert_allclose(new_out, O[0, i, h], rtol=0, atol=1e-30)


# ------------------------------------------------------ planted-mistake checks
# Each entry plants one plausible mistake in a private copy of oracle.c (on the
# CPU; the real oracle is untouched) and requires that the pins above reject it.
_MUTATIONS = {
    "sink dropped from denominator":
        ("double Z = (isinf(sink) && sink < 0) ? 0.0 : exp(sink - M);", "double Z = 0.0;"),
    "sink multiplied by scale":
        ("(double)sinks[h], s,\n                       out + (((int64_t)b",
         "(double)sinks[h] * scale, s,\n                       out + (((int64_t)b"),
    "window one key too wide":
        ("int lo = i - W + 1 < 0 ? 0 : i - W + 1;\n            const uint16_t *qr = q + (((int64_t)b * L + i) * Hq + h) * D;\n            const uint16_t *kb = k + ((int64_t)b * L * Hkv + hk) * D;\n            const uint16_t *vb = v + ((int64_t)b * L * Hkv + hk) * D;\n            attend_row(qr, kb, vb, (int64_t)Hkv * D, lo, i, D, (double)scale,\n                       (double)sinks[h], s,\n                       out",
         "int lo = i - W < 0 ? 0 : i - W;\n            const uint16_t *qr = q + (((int64_t)b * L + i) * Hq + h) * D;\n            const uint16_t *kb = k + ((int64_t)b * L * Hkv + hk) * D;\n            const uint16_t *vb = v + ((int64_t)b * L * Hkv + hk) * D;\n            attend_row(qr, kb, vb, (int64_t)Hkv * D, lo, i, D, (double)scale,\n                       (double)sinks[h], s,\n                       out"),
    "interleaved instead of grouped GQA heads":
        ("    const int group = Hq / Hkv;\n    const int64_t rows = (int64_t)B * L * Hq;",
         "    const int group = 1;\n    const int64_t rows = (int64_t)B * L * Hq;"),
    "values read from the key rows":
        ("const uint16_t *vr = v + (int64_t)(lo + t) * kvstride;",
         "const uint16_t *vr = k + (int64_t)(lo + t) * kvstride;"),
    "output not normalised":
        ("for (int d = 0; d < D; ++d) out[d] /= Z;", ""),
    "LSE without the running max":
        ("*lse = M + log(Z);", "*lse = log(Z);"),
    "exponent sign flipped":
        ("double p = exp(s[t] - M);", "double p = exp(M - s[t]);"),
    "decode window one key short":
        ("int lo = n - W < 0 ? 0 : n - W;", "int lo = n - W + 1 < 0 ? 0 : n - W + 1;"),
    "decode query at position n":
        ("attend_row(q + r * D, kb, vb, (int64_t)Hkv * D, lo, n - 1, D,",
         "attend_row(q + r * D, kb, vb, (int64_t)Hkv * D, lo, n, D,"),
}


def _build_mutant(tmp_path, old, new):
    import ctypes
    import subprocess
    src = open(oracle._SRC).read()
    assert src.count(old) >= 1, "mutation anchor not found in oracle.c"
    path_c = tmp_path / "mutant.c"
    path_c.write_text(src.replace(old, new, 1))
    path_so = tmp_path / "mutant.so"
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                           str(path_c), "-o", str(path_so), "-lm"])
    return str(path_so)


def _pins_for_mutants():
    test_brute_force_dense_sink_column(4, 4, 2, 16)
    test_finite_sink_closed_form(-4, 8)
    test_window_one_closed_form()
    test_decode_matches_dense_last_row()


@pytest.mark.parametrize("name", sorted(_MUTATIONS))
def test_pins_reject_planted_mistake(name, tmp_path, monkeypatch):
    import ctypes
    old, new = _MUTATIONS[name]
    so = _build_mutant(tmp_path, old, new)
    real = oracle._load()
    mutant = ctypes.CDLL(so)
    for fn in ("oracle_num_threads", "oracle_fwd", "oracle_fwd_rows", "oracle_decode",
               "oracle_split_partial", "oracle_combine"):
        getattr(mutant, fn).argtypes = getattr(real, fn).argtypes
        getattr(mutant, fn).restype = getattr(real, fn).restype
    monkeypatch.setattr(oracle, "_lib", mutant)
    with pytest.raises(AssertionError):
        _pins_for_mutants()
