"""GPU parity of the packed variable-length forward (tcgen05 kernel) against the
fp64 oracle.

Bar (the forward's): max|dO| <= 2e-2, max|dLSE| <= 1e-3, no NaN/Inf.  The
packed inputs sit in NaN storage with extra rows after the last sequence, and
the outputs inside NaN guard bands that must come back untouched; every row of
every sequence must be written (ragged last tiles are stored row by row, and a
write into a neighbouring sequence's rows would be caught by the oracle
comparison of that sequence)."""
import numpy as np
import pytest
import torch

import oracle
import sliding_window_learned_b200 as swl
from sliding_window_learned_b200 import inputs

pytestmark = pytest.mark.gpu
TOL_O = 2e-2
TOL_LSE = 1e-3
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sliding_window_learned_b200 import build
    build.build()
    oracle.build()


def _case(lens, Hq, Hkv, D, seed):
    g = torch.Generator().manual_seed(seed)
    T = int(sum(lens))
    q = torch.randn(T, Hq, D, generator=g).bfloat16()
    k = torch.randn(T, Hkv, D, generator=g).bfloat16()
    v = torch.randn(T, Hkv, D, generator=g).bfloat16()
    sinks = torch.rand(Hq, generator=g) * 12.0 - 4.0
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    return q, k, v, cu, sinks


def _in_nan_storage(t, extra=192):
    st = torch.full((t.shape[0] + extra,) + tuple(t.shape[1:]), float("nan"), dtype=t.dtype,
                    device=DEV)
    st[: t.shape[0]] = t.to(DEV)
    return st[: t.shape[0]]


def _guarded(shape, dtype, pad=4096):
    n = int(np.prod(shape))
    buf = torch.full((pad + n + pad,), float("nan"), dtype=dtype, device=DEV)
    return buf[pad:pad + n].view(shape), buf, pad, n


def _gpu(q, k, v, cu, sinks, max_len, W, scale):
    T, Hq, D = q.shape
    out, obuf, oa, on = _guarded((T, Hq, D), torch.bfloat16)
    lse, lbuf, la, ln = _guarded((Hq, T), torch.float32)
    swl.attn_sink_fwd_varlen(_in_nan_storage(q), _in_nan_storage(k), _in_nan_storage(v),
                             cu.to(DEV), max_len, sinks.to(DEV), W, scale, out, lse)
    torch.cuda.synchronize()
    assert swl.attn_sink_get_status() == 0
    for buf, a, n in ((obuf, oa, on), (lbuf, la, ln)):
        assert bool(torch.isnan(buf[:a]).all()) and bool(torch.isnan(buf[a + n:]).all()), "guard written"
    return out.float().cpu().numpy(), lse.cpu().numpy()


def _check(o, lv, ref_o, ref_l, what):
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    assert np.isfinite(lv).all(), f"{what}: non-finite LSE"
    eo = float(np.abs(o - ref_o).max()) if o.size else 0.0
    el = float(np.abs(lv - ref_l).max()) if lv.size else 0.0
    assert eo <= TOL_O, f"{what}: max|dO| = {eo}"
    assert el <= TOL_LSE, f"{what}: max|dLSE| = {el}"


CASES = [  # lens, Hq, Hkv, D, W
    ([1, 127, 128, 129, 300, 0, 513], 8, 2, 128, 1 << 30),
    ([1000, 17, 256, 640], 8, 4, 128, 513),
    ([200, 0, 0, 77, 1], 4, 4, 64, 64),
    ([390, 130], 6, 2, 64, 1),
    ([129, 700], 4, 1, 256, 513),
    ([64, 65, 333], 12, 2, 256, 1 << 30),
    ([1500], 32, 4, 128, 513),
]


@pytest.mark.parametrize("case", CASES, ids=[f"n{len(c[0])}Hq{c[1]}Hkv{c[2]}D{c[3]}W{c[4]}" for c in CASES])
def test_varlen_against_oracle(case):
    lens, Hq, Hkv, D, W = case
    q, k, v, cu, sinks = _case(lens, Hq, Hkv, D, seed=sum(lens) + D)
    scale = 1.0 / np.sqrt(D)
    ref_o, ref_l = oracle.fwd_varlen(inputs.bits(q), inputs.bits(k), inputs.bits(v), cu.numpy(),
                                     sinks.numpy(), W, scale)
    o, lv = _gpu(q, k, v, cu, sinks, max(lens), W, scale)
    _check(o, lv, ref_o, ref_l, f"varlen {lens}")


def test_varlen_matches_batched_forward():
    """Equal lengths: the packed forward and the batched forward of the same
    rows agree (each within the oracle bar; here directly)."""
    B, L, Hq, Hkv, D, W = 3, 700, 8, 2, 128, 513
    q, k, v, cu, sinks = _case([L] * B, Hq, Hkv, D, seed=4)
    scale = 1.0 / np.sqrt(D)
    o, lv = _gpu(q, k, v, cu, sinks, L, W, scale)
    ob, lb = swl.fwd(q.view(B, L, Hq, D).to(DEV), k.view(B, L, Hkv, D).to(DEV),
                     v.view(B, L, Hkv, D).to(DEV), sinks.to(DEV), W, scale)
    torch.cuda.synchronize()
    assert float(np.abs(o - ob.float().cpu().numpy().reshape(B * L, Hq, D)).max()) <= TOL_O
    lb = lb.cpu().numpy().transpose(1, 0, 2).reshape(Hq, B * L)
    assert float(np.abs(lv - lb).max()) <= TOL_LSE


def test_varlen_prefill_mix_sampled():
    """A serving-like mix of 24 sequences of 1 to 4096 tokens at the prefill
    workload's heads (Hq32 Hkv4 D128, W513): every output finite; a sample of
    rows of every sequence (its first, last and a few random ones) against the
    oracle."""
    rng = np.random.default_rng(7)
    lens = [int(x) for x in rng.integers(1, 4097, size=24)]
    Hq, Hkv, D, W = 32, 4, 128, 513
    q, k, v, cu, sinks = _case(lens, Hq, Hkv, D, seed=11)
    scale = 1.0 / np.sqrt(D)
    o, lv = _gpu(q, k, v, cu, sinks, max(lens), W, scale)
    assert np.isfinite(o).all() and np.isfinite(lv).all()
    cun = cu.numpy()
    qb, kb, vb = inputs.bits(q), inputs.bits(k), inputs.bits(v)
    for b, n in enumerate(lens):
        s0 = int(cun[b])
        pos = sorted({0, n - 1, *[int(x) for x in rng.integers(0, n, size=3)]})
        rows = np.array([[0, i, h] for i in pos for h in (0, 13, 31)], np.int32)
        ref_o, ref_l = oracle.fwd_rows(qb[None, s0:s0 + n], kb[None, s0:s0 + n], vb[None, s0:s0 + n],
                                       sinks.numpy(), W, scale, rows)
        got_o = np.stack([o[s0 + i, h] for _, i, h in rows])
        got_l = np.array([lv[h, s0 + i] for _, i, h in rows])
        _check(got_o, got_l, ref_o, ref_l, f"sequence {b} (n={n})")
