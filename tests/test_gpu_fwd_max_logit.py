"""GPU parity of attn_sink_fwd_max_logit: the largest pre-softmax logit of
every (batch, head) against the fp64 oracle (max|d| <= 1e-3, the LSE bar: both
are fp32 functions of the same scores), and O/LSE identical in value to
attn_sink_fwd's."""
import numpy as np
import pytest
import torch

import oracle
import sliding_window_learned_b200 as swl
from sliding_window_learned_b200 import inputs

pytestmark = pytest.mark.gpu
TOL_ML = 1e-3
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sliding_window_learned_b200 import build
    build.build()
    oracle.build()


def _case(B, L, Hq, Hkv, D, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, L, Hq, D, generator=g).bfloat16()
    k = torch.randn(B, L, Hkv, D, generator=g).bfloat16()
    v = torch.randn(B, L, Hkv, D, generator=g).bfloat16()
    sinks = torch.rand(Hq, generator=g) * 12.0 - 4.0
    return q, k, v, sinks


def _run(q, k, v, sinks, W, scale):
    B, L, Hq, D = q.shape
    qd, kd, vd, sd = q.to(DEV), k.to(DEV), v.to(DEV), sinks.to(DEV)
    out = torch.empty_like(qd)
    lse = torch.empty(B, Hq, L, device=DEV)
    ml = torch.full((B + 1, Hq), float("nan"), device=DEV)      # guard row after the output
    swl.attn_sink_fwd_max_logit(qd, kd, vd, sd, W, scale, out, lse, ml[:B])
    ref_o, ref_l = swl.fwd(qd, kd, vd, sd, W, scale)
    torch.cuda.synchronize()
    assert swl.attn_sink_get_status() == 0
    assert bool(torch.isnan(ml[B]).all()), "guard written"
    assert torch.equal(out, ref_o), "O differs from attn_sink_fwd"
    assert torch.equal(lse, ref_l), "LSE differs from attn_sink_fwd"
    return ml[:B].cpu().numpy()


CASES = [  # B, L, Hq, Hkv, D, W
    (1, 256, 4, 2, 64, 64),
    (2, 300, 8, 2, 128, 513),
    (1, 700, 6, 2, 128, 1),
    (2, 517, 4, 4, 64, 1 << 30),
    (1, 400, 4, 2, 256, 129),
    (1, 333, 3, 1, 128, 50),
    (2, 1024, 4, 4, 128, 513),
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}L{c[1]}Hq{c[2]}Hkv{c[3]}D{c[4]}W{c[5]}" for c in CASES])
def test_max_logit_against_oracle(case):
    B, L, Hq, Hkv, D, W = case
    q, k, v, sinks = _case(B, L, Hq, Hkv, D, seed=L + D)
    scale = 1.0 / np.sqrt(D)
    got = _run(q, k, v, sinks, W, scale)
    ref = oracle.max_logit(inputs.bits(q), inputs.bits(k), W, scale)
    assert np.isfinite(got).all()
    assert float(np.abs(got - ref).max()) <= TOL_ML


def test_max_logit_prefill_workload():
    """The prefill workload (B2 Hq32 Hkv4 L4096 D128 W513): all 64 maxima
    finite; those of the first kv group's 8 heads against the oracle."""
    cfg = inputs.PREFILL
    x = inputs.make_prefill(cfg, seed=0)
    got = _run(x["q"], x["k"], x["v"], x["sinks"], cfg.W, cfg.scale)
    assert np.isfinite(got).all()
    ref = oracle.max_logit(inputs.bits(x["q"][:, :, :8]), inputs.bits(x["k"][:, :, :1]), cfg.W, cfg.scale)
    assert float(np.abs(got[:, :8] - ref).max()) <= TOL_ML
