"""Seeded random sweep against the fp64 oracle: forward, decode and backward on
shapes drawn from one fixed seed (head dims, GQA group sizes including odd ones,
windows from 1 to past the end, ragged lengths, sinks from absent to far above
the logits), each at the bar of its dedicated test: forward max|dO| <= 2e-2 and
max|dLSE| <= 1e-3, decode max|dO| <= 2e-2, backward max|d| <= 2e-2 * max(1,
max|ref|) per gradient.  The draws are sized so that the oracle finishes each
case in about a second."""
import numpy as np
import pytest
import torch

import oracle
import sliding_window_learned_b200 as swl
from sliding_window_learned_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"
_RNG = np.random.default_rng(2026)


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sliding_window_learned_b200 import build
    build.build()
    oracle.build()


def _sinks(kind, Hq, g):
    if kind == "none":
        return torch.full((Hq,), float("-inf"))
    if kind == "high":
        return torch.full((Hq,), 12.0) + torch.rand(Hq, generator=g)
    if kind == "low":
        return torch.full((Hq,), -30.0) + torch.rand(Hq, generator=g)
    return torch.rand(Hq, generator=g) * 12.0 - 4.0


def _window(L, r):
    return int([1, r.integers(2, 40), max(1, L // 2), L, 1 << 30][r.integers(0, 5)])


def _draw(n, max_work, max_L, dims, with_hkv_cap=8):
    out = []
    while len(out) < n:
        D = int(dims[_RNG.integers(0, len(dims))])
        Hkv = int([1, 2, 4][_RNG.integers(0, 3)])
        G = int([1, 2, 3, 4, 8][_RNG.integers(0, 5)])
        Hq = Hkv * G
        B = int(_RNG.integers(1, 4))
        L = int(_RNG.integers(1, max_L + 1))
        W = _window(L, _RNG)
        if Hq > 16 or Hkv > with_hkv_cap or B * L * Hq * min(L, W) * D > max_work:
            continue
        sink = ["uniform", "none", "high", "low"][_RNG.integers(0, 4)]
        out.append((B, L, Hq, Hkv, D, W, sink, int(_RNG.integers(0, 1 << 30))))
    return out


FWD = _draw(20, 4e8, 600, (64, 128, 256))
BWD = _draw(10, 1.5e8, 300, (64, 128))


def _case(B, L, Hq, Hkv, D, seed, sink):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, L, Hq, D, generator=g).bfloat16()
    k = torch.randn(B, L, Hkv, D, generator=g).bfloat16()
    v = torch.randn(B, L, Hkv, D, generator=g).bfloat16()
    do = torch.randn(B, L, Hq, D, generator=g).bfloat16()
    return q, k, v, do, _sinks(sink, Hq, g)


@pytest.mark.parametrize("c", FWD, ids=[f"B{c[0]}L{c[1]}Hq{c[2]}Hkv{c[3]}D{c[4]}W{c[5]}{c[6]}" for c in FWD])
def test_forward_sweep(c):
    B, L, Hq, Hkv, D, W, sink, seed = c
    q, k, v, _, s = _case(B, L, Hq, Hkv, D, seed, sink)
    scale = D ** -0.5
    ref_o, ref_l = oracle.fwd(inputs.bits(q), inputs.bits(k), inputs.bits(v), s.numpy(), W, scale)
    o, lse = swl.fwd(q.to(DEV), k.to(DEV), v.to(DEV), s.to(DEV), W, scale)
    torch.cuda.synchronize()
    assert swl.attn_sink_get_status() == 0
    o, lse = o.float().cpu().numpy(), lse.cpu().numpy()
    assert np.isfinite(o).all()
    assert float(np.abs(o - ref_o).max()) <= 2e-2
    fin = np.isfinite(ref_l)
    assert (np.isfinite(lse) == fin).all()
    assert float(np.abs(lse[fin] - ref_l[fin]).max(initial=0.0)) <= 1e-3


DEC = []
while len(DEC) < 12:
    D = int([64, 128, 256][_RNG.integers(0, 3)])
    Hkv = int([1, 2, 4][_RNG.integers(0, 3)])
    G = int([1, 2, 4, 8, 16][_RNG.integers(0, 5)])
    if Hkv * G > 32 or (D == 256 and G > 8):        # (the decode's documented limits)
        continue
    B = int(_RNG.integers(1, 5))
    Smax = int(_RNG.integers(1, 2049))
    lens = [int(x) for x in _RNG.integers(0, Smax + 1, size=B)]
    W = _window(Smax, _RNG)
    DEC.append((B, Smax, Hkv * G, Hkv, D, W, lens, ["uniform", "none", "high", "low"][_RNG.integers(0, 4)],
                int(_RNG.integers(0, 1 << 30))))


@pytest.mark.parametrize("c", DEC, ids=[f"B{c[0]}S{c[1]}Hq{c[2]}Hkv{c[3]}D{c[4]}W{c[5]}{c[7]}" for c in DEC])
def test_decode_sweep(c):
    B, Smax, Hq, Hkv, D, W, lens, sink, seed = c
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, D, generator=g).bfloat16()
    kc = torch.randn(B, Smax, Hkv, D, generator=g).bfloat16()
    vc = torch.randn(B, Smax, Hkv, D, generator=g).bfloat16()
    for b, n in enumerate(lens):                     # past each end: NaN, so a read shows up
        kc[b, n:] = float("nan")
        vc[b, n:] = float("nan")
    s = _sinks(sink, Hq, g)
    sl = torch.tensor(lens, dtype=torch.int32)
    scale = D ** -0.5
    ref, _ = oracle.decode(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), sl.numpy(), s.numpy(), W, scale)
    out = swl.decode(q.to(DEV), kc.to(DEV), vc.to(DEV), sl.to(DEV), s.to(DEV), W, scale)
    torch.cuda.synchronize()
    assert swl.attn_sink_get_status() == 0
    o = out.float().cpu().numpy()
    assert np.isfinite(o).all()
    assert float(np.abs(o - ref).max()) <= 2e-2


@pytest.mark.parametrize("c", BWD, ids=[f"B{c[0]}L{c[1]}Hq{c[2]}Hkv{c[3]}D{c[4]}W{c[5]}{c[6]}" for c in BWD])
def test_backward_sweep(c):
    B, L, Hq, Hkv, D, W, sink, seed = c
    q, k, v, do, s = _case(B, L, Hq, Hkv, D, seed, sink)
    scale = D ** -0.5
    ref = oracle.bwd(inputs.bits(q), inputs.bits(k), inputs.bits(v), s.numpy(), inputs.bits(do), W, scale)
    qd, kd, vd, sd = q.to(DEV), k.to(DEV), v.to(DEV), s.to(DEV)
    o, lse = swl.fwd(qd, kd, vd, sd, W, scale)
    grads = [torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd), torch.empty(Hq, device=DEV)]
    swl.attn_sink_bwd(qd, kd, vd, o, lse, do.to(DEV), sd, W, scale, *grads)
    torch.cuda.synchronize()
    assert swl.attn_sink_get_status() == 0
    for name, got, r in zip(("dq", "dk", "dv", "dsink"), grads, ref[:4]):
        gn = got.float().cpu().numpy()
        assert np.isfinite(gn).all(), name
        assert float(np.abs(gn - r).max()) <= 2e-2 * max(1.0, float(np.abs(r).max())), name
