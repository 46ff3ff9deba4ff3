"""Error paths, exercised without a GPU fault.

A device wait that runs out.  With the wait limit set to a few nanoseconds
(attn_sink_set_wait_limit_ns), the first wait of a small forward, decode or
backward call that is not satisfied at once gives up: its CTA stops issuing
work, lets the copies and tensor-core operations it already started finish,
frees its tensor memory and returns, and the call leaves ATTN_ETIMEOUT in the
device status word.  The limit only shortens waits that would have completed:
no barrier is left short of arrivals and nothing waits forever (the page
"cf-1.com/news/6055759", "fix 1", describes the hang that a barrier missing a
participant causes; every wait here is bounded so that such a fault ends in a
status code).  The next call, with the default limit, is exact again.

A workspace allocation that fails.  Injected on the host
(attn_sink_fail_workspace_allocs): the call returns ATTN_ENOMEM and launches
nothing, so its output buffer keeps its NaN fill.
"""
import numpy as np
import pytest
import torch

import oracle
import sliding_window_learned_b200 as swl
from sliding_window_learned_b200 import abi, inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL_O, TOL_LSE = 2e-2, 1e-3


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sliding_window_learned_b200 import build
    build.build()
    oracle.build()
    yield
    swl.attn_sink_set_wait_limit_ns(0)
    swl.attn_sink_fail_workspace_allocs(0)


def _timed_out(call):
    """Run `call` with a 1 ns wait limit, L2 flushed first (so its first
    copies come from DRAM); return the status code it left."""
    torch.cuda.synchronize()
    assert swl.attn_sink_get_status() == 0
    torch.empty(64 << 20, device=DEV).fill_(1.0)
    swl.attn_sink_set_wait_limit_ns(1)
    try:
        call()
        torch.cuda.synchronize()
        return swl.attn_sink_get_status()
    finally:
        swl.attn_sink_set_wait_limit_ns(0)


# (B, L, Hq, Hkv, D, W): head dims 64, 128 and 256 of the tensor-core kernel,
# with groups of 2 and 3 query heads and two kv heads
FWD_CASES = [(1, 128, 2, 1, 64, 64), (1, 200, 3, 1, 128, 100), (1, 130, 2, 2, 256, 64)]


@pytest.mark.parametrize("case", FWD_CASES, ids=[f"Hq{c[2]}Hkv{c[3]}D{c[4]}" for c in FWD_CASES])
def test_forward_wait_runs_out_then_recovers(case):
    B, L, Hq, Hkv, D, W = case
    cfg = inputs.Prefill("case", B, L, Hq, Hkv, D, W, ("uniform", -4, 8))
    x = inputs.make_prefill(cfg, seed=L + D)
    q, k, v, s = (x[n].to(DEV) for n in ("q", "k", "v", "sinks"))
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, L, device=DEV)
    rc = _timed_out(lambda: swl.attn_sink_fwd(q, k, v, s, W, cfg.scale, out, lse))
    assert rc == abi.ATTN_ETIMEOUT, rc
    # the status word was cleared by the read; the next call is exact
    assert swl.attn_sink_get_status() == 0
    out.fill_(float("nan"))
    swl.attn_sink_fwd(q, k, v, s, W, cfg.scale, out, lse)
    torch.cuda.synchronize()
    assert swl.attn_sink_get_status() == 0
    ref_o, ref_l = oracle.fwd(inputs.bits(x["q"]), inputs.bits(x["k"]), inputs.bits(x["v"]),
                              x["sinks"].numpy(), W, cfg.scale)
    assert float(np.abs(out.float().cpu().numpy() - ref_o).max()) <= TOL_O
    assert float(np.abs(lse.cpu().numpy() - ref_l).max()) <= TOL_LSE


def _decode_case(seed=7, B=4, Smax=16384, lens=(16384, 9000, 5000, 12345)):
    g = torch.Generator().manual_seed(seed)
    Hq, Hkv, D = 8, 2, 128
    q = torch.randn(B, Hq, D, generator=g).bfloat16()
    kc = torch.randn(B, Smax, Hkv, D, generator=g).bfloat16()
    vc = torch.randn(B, Smax, Hkv, D, generator=g).bfloat16()
    sl = torch.tensor(lens[:B], dtype=torch.int32)
    s = torch.rand(Hq, generator=g) * 12 - 4
    return q, kc, vc, sl, s


def test_decode_wait_runs_out_then_recovers():
    q, kc, vc, sl, s = _decode_case()
    dq, dk, dv, dsl, ds = (t.to(DEV) for t in (q, kc, vc, sl, s))
    scale = 1.0 / np.sqrt(q.shape[-1])
    out = torch.empty_like(dq)
    rc = _timed_out(lambda: swl.attn_sink_decode(dq, dk, dv, dsl, ds, 1 << 30, scale, out))
    assert rc == abi.ATTN_ETIMEOUT, rc
    assert swl.attn_sink_get_status() == 0
    out.fill_(float("nan"))
    swl.attn_sink_decode(dq, dk, dv, dsl, ds, 1 << 30, scale, out)
    torch.cuda.synchronize()
    assert swl.attn_sink_get_status() == 0
    ref = oracle.decode(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), sl.numpy(), s.numpy(), 1 << 30,
                        scale)[0]
    assert float(np.abs(out.float().cpu().numpy() - ref).max()) <= TOL_O


def _bwd_case():
    g = torch.Generator().manual_seed(11)
    B, L, Hq, Hkv, D, W = 1, 256, 2, 1, 128, 100
    q = torch.randn(B, L, Hq, D, generator=g).bfloat16()
    k = torch.randn(B, L, Hkv, D, generator=g).bfloat16()
    v = torch.randn(B, L, Hkv, D, generator=g).bfloat16()
    do = torch.randn(B, L, Hq, D, generator=g).bfloat16()
    s = torch.rand(Hq, generator=g) * 12 - 4
    return q, k, v, do, s, W


def test_backward_wait_runs_out_then_recovers():
    q, k, v, do, s, W = _bwd_case()
    scale = 1.0 / np.sqrt(q.shape[-1])
    ref = oracle.bwd(inputs.bits(q), inputs.bits(k), inputs.bits(v), s.numpy(), inputs.bits(do), W, scale)
    dq_, dk_, dv_, ddo, ds = (t.to(DEV) for t in (q, k, v, do, s))
    o = torch.from_numpy(ref[4]).float().to(DEV)
    lse = torch.from_numpy(ref[5]).float().to(DEV)
    grads = [torch.empty_like(dq_), torch.empty_like(dk_), torch.empty_like(dv_),
             torch.empty(q.shape[2], device=DEV)]

    def call():
        swl.attn_sink_bwd(dq_, dk_, dv_, o, lse, ddo, ds, W, scale, *grads)

    rc = _timed_out(call)
    assert rc == abi.ATTN_ETIMEOUT, rc
    assert swl.attn_sink_get_status() == 0
    call()
    torch.cuda.synchronize()
    assert swl.attn_sink_get_status() == 0
    for got, want in zip(grads[:3], ref[:3]):
        g = got.float().cpu().numpy()
        assert np.isfinite(g).all()
        assert float(np.abs(g - want).max()) <= 2e-2 * max(1.0, float(np.abs(want).max()))


def test_workspace_allocation_failure_launches_nothing():
    q, kc, vc, sl, s = _decode_case(seed=3, B=2, Smax=300, lens=(300, 131))
    dq, dk, dv, dsl, ds = (t.to(DEV) for t in (q, kc, vc, sl, s))
    scale = 1.0 / np.sqrt(q.shape[-1])
    torch.cuda.synchronize()
    out = torch.full_like(dq, float("nan"))
    swl.attn_sink_fail_workspace_allocs(1)
    try:
        with pytest.raises(swl.AttnSinkError) as err:
            swl.attn_sink_decode(dq, dk, dv, dsl, ds, 1 << 30, scale, out)
        assert err.value.code == abi.ATTN_ENOMEM
    finally:
        swl.attn_sink_fail_workspace_allocs(0)
    torch.cuda.synchronize()
    assert swl.attn_sink_get_status() == 0
    assert bool(torch.isnan(out.float()).all()), "a kernel ran although the allocation failed"
    # the same for the backward's workspace, then a normal call
    qb, kb, vb, dob, sb, W = _bwd_case()
    grads = [torch.full_like(qb, float("nan"), device=DEV), torch.full_like(kb, float("nan"), device=DEV),
             torch.full_like(vb, float("nan"), device=DEV), torch.full((qb.shape[2],), float("nan"), device=DEV)]
    o = torch.zeros(qb.shape, device=DEV)
    lse = torch.zeros(qb.shape[0], qb.shape[2], qb.shape[1], device=DEV)
    swl.attn_sink_fail_workspace_allocs(1)
    try:
        with pytest.raises(swl.AttnSinkError) as err:
            swl.attn_sink_bwd(qb.to(DEV), kb.to(DEV), vb.to(DEV), o, lse, dob.to(DEV), sb.to(DEV), W,
                              1.0 / np.sqrt(qb.shape[-1]), *grads)
        assert err.value.code == abi.ATTN_ENOMEM
    finally:
        swl.attn_sink_fail_workspace_allocs(0)
    torch.cuda.synchronize()
    assert all(bool(torch.isnan(t.float()).all()) for t in grads)
    swl.attn_sink_decode(dq, dk, dv, dsl, ds, 1 << 30, scale, out)
    torch.cuda.synchronize()
    assert swl.attn_sink_get_status() == 0
    assert torch.isfinite(out.float()).all()
