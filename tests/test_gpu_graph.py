"""The C-ABI calls under CUDA-graph stream capture: attn_sink_fwd,
attn_sink_decode (plan, split and combine, with its workspace taken from the
stream-ordered pool inside the capture) and attn_sink_bwd are captured once,
the input buffers are refilled, and each replay must equal the eager call on
the same inputs bit for bit."""
import pytest
import torch

import sliding_window_learned_b200 as swl
from sliding_window_learned_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sliding_window_learned_b200 import build
    build.build()


def _fill(bufs, seed):
    g = torch.Generator(device=DEV).manual_seed(seed)
    for t in bufs:
        t.copy_(torch.randn(t.shape, device=DEV, generator=g).to(t.dtype))


def test_forward_decode_backward_replay_equal_eager():
    B, L, Hq, Hkv, D, W = 2, 700, 8, 2, 128, 129
    scale = D ** -0.5
    q = torch.empty(B, L, Hq, D, dtype=torch.bfloat16, device=DEV)
    k = torch.empty(B, L, Hkv, D, dtype=torch.bfloat16, device=DEV)
    v = torch.empty_like(k)
    do = torch.empty_like(q)
    sinks = torch.empty(Hq, device=DEV)
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, L, device=DEV)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dsink = torch.empty(Hq, device=DEV)
    # decode over the same K/V as a cache, the last query row as the token
    qd = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=DEV)
    seqlens = torch.tensor([L, L // 3], dtype=torch.int32, device=DEV)
    od = torch.empty_like(qd)

    def step(stream=None):
        swl.attn_sink_fwd(q, k, v, sinks, W, scale, o, lse, stream)
        swl.attn_sink_bwd(q, k, v, o, lse, do, sinks, W, scale, dq, dk, dv, dsink, stream)
        swl.attn_sink_decode(qd, k, v, seqlens, sinks, W, scale, od, stream)

    _fill([q, k, v, do, sinks, qd], seed=1)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):                      # warm up outside the capture
        step(s)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        step(s)
    torch.cuda.synchronize()
    assert swl.attn_sink_get_status() == 0
    for seed in (2, 3):
        _fill([q, k, v, do, sinks, qd], seed=seed)
        graph.replay()
        torch.cuda.synchronize()
        got = [t.clone() for t in (o, lse, dq, dk, dv, dsink, od)]
        step()                                      # eager on the same inputs
        torch.cuda.synchronize()
        assert swl.attn_sink_get_status() == 0
        want = [o, lse, dq, dk, dv, dsink, od]
        for name, a, b in zip(("o", "lse", "dq", "dk", "dv", "dsink", "decode o"), got, want):
            assert torch.isfinite(a.float()).all(), name
            if name in ("dq", "dk", "dv", "dsink"):
                # fp32 atomic sums: the order of additions may differ between runs
                tol = 1e-2 * max(1.0, float(b.float().abs().max()))
                assert float((a.float() - b.float()).abs().max()) <= tol, name
            else:
                assert torch.equal(a, b), name
