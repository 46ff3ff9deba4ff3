"""GPU parity of the prefill forward (tcgen05 kernel, and the CUDA-core second
implementation) against the fp64 oracle on the same seeded bf16 inputs.

Bar: max|dO| <= 2e-2 and max|dLSE| <= 1e-3 over every compared element, and no
NaN/Inf anywhere in the outputs.  Output buffers sit inside NaN-filled guard
bands that must come back untouched; inputs are views into larger NaN-filled
storage, so a read past the end of a sequence would show up as NaN."""

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


def _guarded(shape, dtype, pad_front=4096, pad_back=4096):
    """A tensor of `shape` inside a NaN-filled flat buffer; returns (view, buffer, offset)."""
    n = int(np.prod(shape))
    buf = torch.full((pad_front + n + pad_back,), float("nan"), dtype=dtype, device=DEV)
    view = buf[pad_front:pad_front + n].view(shape)
    return view, buf, (pad_front, n)


def _guard_intact(buf, span):
    a, n = span
    head = buf[:a]
    tail = buf[a + n:]
    return bool(torch.isnan(head).all()) and bool(torch.isnan(tail).all())


def _padded_input(t, extra_rows=64):
    """Place t [B,L,H,D] in NaN storage with extra positions after L."""
    B, L, H, D = t.shape
    st = torch.full((B, L + extra_rows, H, D), float("nan"), dtype=t.dtype, device=DEV)
    st[:, :L] = t.to(DEV)
    return st[:, :L]


def run_gpu(x, window, scale, impl="tc", with_lse=True):
    q = _padded_input(x["q"])
    k = _padded_input(x["k"])
    v = _padded_input(x["v"])
    sinks = x["sinks"].to(DEV)
    B, L, Hq, D = q.shape
    out, obuf, ospan = _guarded((B, L, Hq, D), torch.bfloat16)
    lse, lbuf, lspan = _guarded((B, Hq, L), torch.float32) if with_lse else (None, None, None)
    fn = swl.attn_sink_fwd if impl == "tc" else swl.attn_sink_fwd_cudacore
    fn(q, k, v, sinks, window, scale, out, lse)
    torch.cuda.synchronize()
    assert swl.attn_sink_get_status() == 0
    assert _guard_intact(obuf, ospan), "write outside the output tensor"
    if with_lse:
        assert _guard_intact(lbuf, lspan), "write outside the LSE tensor"
    o = out.float().cpu().numpy()
    lv = lse.cpu().numpy() if with_lse else None
    return o, lv


def check(o, lv, ref_o, ref_l, what=""):
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    err_o = float(np.abs(o - ref_o).max()) if o.size else 0.0
    assert err_o <= TOL_O, f"{what}: max|dO| = {err_o}"
    if lv is not None:
        assert np.isfinite(lv).all(), f"{what}: non-finite LSE"
        err_l = float(np.abs(lv - ref_l).max()) if lv.size else 0.0
        assert err_l <= TOL_LSE, f"{what}: max|dLSE| = {err_l}"


def oracle_fwd(x, window, scale):
    return oracle.fwd(inputs.bits(x["q"]), inputs.bits(x["k"]), inputs.bits(x["v"]),
                      x["sinks"].numpy(), window, scale)


@pytest.mark.parametrize("impl", ["tc", "cudacore"])
def test_tiny_workload(impl):
    cfg = inputs.TINY
    x = inputs.make_prefill(cfg, seed=0)
    ref_o, ref_l = oracle_fwd(x, cfg.W, cfg.scale)
    o, lv = run_gpu(x, cfg.W, cfg.scale, impl)
    check(o, lv, ref_o, ref_l, f"tiny/{impl}")


# (B, L, Hq, Hkv, D, W, sinks) -- ragged L, windows around tile edges, GQA 1..8
CASES = [
    (1, 1, 2, 1, 64, 1, ("uniform", -4, 8)),
    (1, 77, 4, 4, 64, 3, ("uniform", -4, 8)),
    (2, 129, 4, 2, 64, 127, ("uniform", -4, 8)),
    (1, 300, 8, 1, 64, 129, ("normal", 0, 2)),
    (1, 128, 2, 2, 128, 128, ("uniform", -4, 8)),
    (1, 257, 8, 2, 128, 2, ("uniform", -4, 8)),
    (2, 700, 8, 1, 128, 513, ("uniform", -4, 8)),
    (1, 1000, 4, 4, 128, 100000, ("normal", 0, 2)),
    (1, 385, 16, 2, 128, 1, ("const", float("-inf"))),
    (1, 640, 4, 1, 128, 256, ("const", 30.0)),
    (1, 200, 2, 2, 256, 64, ("uniform", -4, 8)),
    (1, 513, 4, 2, 256, 513, ("split", 20.0, -50.0)),
    (2, 333, 8, 8, 256, 1000, ("normal", 0, 2)),
    (1, 64, 2, 1, 256, 1, ("uniform", -4, 8)),
    # one query head per kv head, or an odd group: the one-head kernel, over
    # several query tiles with ragged tails
    (2, 1000, 4, 4, 128, 513, ("uniform", -4, 8)),
    (1, 512, 3, 1, 128, 1, ("uniform", -4, 8)),
    (1, 768, 6, 2, 128, 129, ("normal", 0, 2)),
    (2, 256, 2, 2, 64, 200, ("uniform", -4, 8)),
    (1, 900, 4, 4, 64, 300, ("const", 30.0)),
    (1, 640, 4, 4, 128, 513, ("uniform", -4, 8)),
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}L{c[1]}Hq{c[2]}Hkv{c[3]}D{c[4]}W{c[5]}-{c[6][0]}"
                                             for c in CASES])
def test_shapes_against_oracle(case):
    B, L, Hq, Hkv, D, W, sk = case
    cfg = inputs.Prefill("case", B, L, Hq, Hkv, D, W, sk)
    x = inputs.make_prefill(cfg, seed=L + D)
    ref_o, ref_l = oracle_fwd(x, W, cfg.scale)
    o, lv = run_gpu(x, W, cfg.scale, "tc")
    check(o, lv, ref_o, ref_l, "tc")


def test_lse_optional_and_scale_not_inverse_sqrt():
    cfg = inputs.Prefill("case", 1, 300, 4, 2, 128, 200, ("uniform", -4, 8))
    x = inputs.make_prefill(cfg, seed=5)
    scale = 0.3
    ref_o, _ = oracle_fwd(x, cfg.W, scale)
    o, lv = run_gpu(x, cfg.W, scale, "tc", with_lse=False)
    assert lv is None
    check(o, None, ref_o, None, "no-lse")


def test_strided_packed_qkv():
    """q, k, v as head-slices of one packed [B, L, Hq+2Hkv, D] projection."""
    B, L, Hq, Hkv, D, W = 1, 400, 8, 2, 128, 130
    cfg = inputs.Prefill("case", B, L, Hq, Hkv, D, W, ("uniform", -4, 8))
    x = inputs.make_prefill(cfg, seed=9)
    packed = torch.cat([x["q"], x["k"], x["v"]], dim=2).to(DEV)
    q, k, v = packed[:, :, :Hq], packed[:, :, Hq:Hq + Hkv], packed[:, :, Hq + Hkv:]
    out = torch.empty(B, L, Hq, D, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(B, Hq, L, dtype=torch.float32, device=DEV)
    swl.attn_sink_fwd(q, k, v, x["sinks"].to(DEV), W, cfg.scale, out, lse)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle_fwd(x, W, cfg.scale)
    check(out.float().cpu().numpy(), lse.cpu().numpy(), ref_o, ref_l, "packed")


def test_empty_sequence_is_noop():
    q = torch.empty(1, 0, 4, 64, dtype=torch.bfloat16, device=DEV)
    k = torch.empty(1, 0, 2, 64, dtype=torch.bfloat16, device=DEV)
    s = torch.zeros(4, device=DEV)
    out = torch.empty_like(q)
    swl.attn_sink_fwd(q, k, k, s, 8, 0.125, out, None)
    torch.cuda.synchronize()


def test_tc_matches_cudacore_bitwise_close_on_random():
    """The two GPU implementations agree with each other (both vs oracle above)."""
    cfg = inputs.Prefill("case", 1, 1024, 8, 2, 128, 513, ("uniform", -4, 8))
    x = inputs.make_prefill(cfg, seed=13)
    a, la = run_gpu(x, cfg.W, cfg.scale, "tc")
    b, lb = run_gpu(x, cfg.W, cfg.scale, "cudacore")
    assert float(np.abs(a - b).max()) <= TOL_O and float(np.abs(la - lb).max()) <= TOL_LSE


# ------------------------------------------------------ full-size workloads
def test_prefill_workload_full():
    """B2 Hq32 Hkv4 L4096 D128 W513: every output against the oracle."""
    cfg = inputs.PREFILL
    x = inputs.make_prefill(cfg, seed=0)
    o, lv = run_gpu(x, cfg.W, cfg.scale, "tc")
    ref_o, ref_l = oracle_fwd(x, cfg.W, cfg.scale)
    check(o, lv, ref_o, ref_l, "prefill")


def test_stress_workload_full():
    """B1 Hq16 Hkv2 L8192 D256 W513, content logits near -150, sinks +20 / -50:
    finite and equal to the oracle everywhere."""
    cfg = inputs.STRESS
    x = inputs.make_prefill(cfg, seed=0)
    o, lv = run_gpu(x, cfg.W, cfg.scale, "tc")
    ref_o, ref_l = oracle_fwd(x, cfg.W, cfg.scale)
    check(o, lv, ref_o, ref_l, "stress")
    # the +20 heads are sink-dominated: |O| is astronomically small, LSE = sink
    assert np.abs(o[:, :, :8]).max() < 1e-30
    np.testing.assert_allclose(lv[:, :8], 20.0, atol=TOL_LSE)


def test_long_causal_workload_full():
    """B1 Hq32 Hkv8 L16384 D128 full causal (2.2 TFLOP): every output and LSE
    against the fp64 oracle (about a minute and a half of oracle time on 16
    host cores), plus the probability-mass bound |O| <= max|v|."""
    cfg = inputs.LONG_CAUSAL
    x = inputs.make_prefill(cfg, seed=0)
    o, lv = run_gpu(x, cfg.W, cfg.scale, "tc")
    ref_o, ref_l = oracle_fwd(x, cfg.W, cfg.scale)
    check(o, lv, ref_o, ref_l, "long-causal")
    vmax = float(x["v"].float().abs().max())
    assert np.abs(o).max() <= vmax + TOL_O
