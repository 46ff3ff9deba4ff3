"""GPU parity of the split-KV decode (plan + split + combine kernels) against
the fp64 oracle.  Cache slots at positions >= seqlens[b] hold bf16 NaN, so any
read past a sequence's end shows up in the output.  Bar: max|dO| <= 2e-2, no
NaN/Inf."""
import numpy as np
import pytest
import torch

import oracle
import sliding_window_learned_b200 as swl
from sliding_window_learned_b200 import inputs

pytestmark = pytest.mark.gpu
TOL_O = 2e-2
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sliding_window_learned_b200 import build
    build.build()
    oracle.build()


def _decode_inputs(B, Smax, Hq, Hkv, D, seqlens, seed, sinks=("uniform", -4.0, 8.0)):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, D, generator=g).bfloat16()
    kc = torch.randn(B, Smax, Hkv, D, generator=g).bfloat16()
    vc = torch.randn(B, Smax, Hkv, D, generator=g).bfloat16()
    for b, n in enumerate(seqlens):
        kc[b, n:] = float("nan")
        vc[b, n:] = float("nan")
    if sinks[0] == "uniform":
        s = torch.rand(Hq, generator=g) * (sinks[2] - sinks[1]) + sinks[1]
    else:
        s = torch.full((Hq,), float(sinks[1]))
    return q, kc, vc, torch.tensor(seqlens, dtype=torch.int32), s


def _oracle(q, kc, vc, sl, s, W, scale):
    return oracle.decode(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), sl.numpy(),
                         s.numpy(), W, scale)[0]


def _gpu(q, kc, vc, sl, s, W, scale, chunk=0):
    out = torch.full((q.shape[0] + 2,) + tuple(q.shape[1:]), float("nan"), dtype=torch.bfloat16,
                     device=DEV)
    o = out[1:-1]
    swl.attn_sink_decode_chunked(q.to(DEV), kc.to(DEV), vc.to(DEV), sl.to(DEV), s.to(DEV), W,
                                 scale, chunk, o)
    torch.cuda.synchronize()
    assert swl.attn_sink_get_status() == 0
    assert bool(torch.isnan(out[0]).all()) and bool(torch.isnan(out[-1]).all()), "guard written"
    return o.float().cpu().numpy()


def _check(o, ref, what):
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    err = float(np.abs(o - ref).max())
    assert err <= TOL_O, f"{what}: max|dO| = {err}"


CASES = [  # B, Smax, Hq, Hkv, D, W, seqlens
    (5, 300, 8, 2, 128, 1 << 30, [1, 63, 64, 65, 300]),
    (3, 1000, 8, 1, 128, 100, [0, 1000, 517]),
    (4, 640, 32, 4, 128, 640, [640, 1, 2, 129]),
    (2, 500, 4, 4, 64, 1, [500, 37]),
    (2, 700, 16, 1, 64, 256, [700, 300]),
    (2, 400, 16, 1, 128, 1 << 30, [399, 400]),
    (3, 333, 8, 2, 256, 1 << 30, [333, 100, 0]),
    (2, 1024, 6, 2, 256, 513, [1024, 600]),
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}S{c[1]}Hq{c[2]}Hkv{c[3]}D{c[4]}W{c[5]}" for c in CASES])
@pytest.mark.parametrize("chunk", [0, 64])
def test_decode_against_oracle(case, chunk):
    B, Smax, Hq, Hkv, D, W, sl = case
    q, kc, vc, sl_t, s = _decode_inputs(B, Smax, Hq, Hkv, D, sl, seed=Smax + D)
    scale = 1.0 / np.sqrt(D)
    ref = _oracle(q, kc, vc, sl_t, s, W, scale)
    o = _gpu(q, kc, vc, sl_t, s, W, scale, chunk)
    _check(o, ref, f"decode chunk={chunk}")


@pytest.mark.parametrize("nsplits", [1, 2, 31, 32, 33, 70])
def test_forced_split_counts(nsplits):
    """One long sequence split into exactly n chunks (and a short one with
    fewer), all agreeing with the unsplit oracle: the combine reduces only the
    splits that exist; 33 and 70 take the general (> 32 splits) path."""
    chunk = 64
    n_long = chunk * nsplits - 17 if nsplits > 1 else 50
    Smax = max(n_long, 200)
    q, kc, vc, sl_t, s = _decode_inputs(2, Smax, 8, 1, 128, [n_long, 130], seed=nsplits)
    scale = 1.0 / np.sqrt(128)
    ref = _oracle(q, kc, vc, sl_t, s, 1 << 30, scale)
    o = _gpu(q, kc, vc, sl_t, s, 1 << 30, scale, chunk)
    _check(o, ref, f"{nsplits} splits")


def test_sink_minus_inf_and_dominant_sink():
    for sk in (("const", float("-inf")), ("const", 40.0)):
        q, kc, vc, sl_t, s = _decode_inputs(3, 256, 8, 2, 128, [256, 10, 1], seed=3, sinks=sk)
        scale = 1.0 / np.sqrt(128)
        ref = _oracle(q, kc, vc, sl_t, s, 1 << 30, scale)
        o = _gpu(q, kc, vc, sl_t, s, 1 << 30, scale, 64)
        _check(o, ref, f"sinks {sk}")


def test_decode_workload_full():
    """B64 Hq32 Hkv4 D128, lengths ~ U[4096, 131072] (generated on the device):
    every output of all 64 sequences against the fp64 oracle, one sequence at
    a time (only its valid prefix of the cache comes to the host)."""
    cfg = inputs.DECODE
    y = inputs.make_decode(cfg, seed=0, device=DEV)
    out = torch.empty_like(y["q"])
    swl.attn_sink_decode(y["q"], y["kcache"], y["vcache"], y["seqlens"], y["sinks"], cfg.W,
                         cfg.scale, out)
    torch.cuda.synchronize()
    assert swl.attn_sink_get_status() == 0
    o = out.float().cpu().numpy()
    assert np.isfinite(o).all()
    sl = y["seqlens"].cpu().numpy()
    sinks = y["sinks"].cpu().numpy()
    worst = 0.0
    for b in range(cfg.B):
        n = int(sl[b])
        ref = oracle.decode(inputs.bits(y["q"][b:b + 1]), inputs.bits(y["kcache"][b:b + 1, :n]),
                            inputs.bits(y["vcache"][b:b + 1, :n]), np.array([n], np.int32),
                            sinks, cfg.W, cfg.scale)[0]
        _check(o[b:b + 1], ref, f"decode seq {b} (n={n})")
        worst = max(worst, float(np.abs(o[b:b + 1] - ref).max()))
    assert worst <= TOL_O
