"""attn_sink_decode_noalloc: the decode entry point for callers that may not
allocate device memory while decoding (engines that reserve nearly all of HBM
for their KV cache up front, or runtimes whose allocator owns every device
byte).  Its workspace is the library's fixed device array instead of a
stream-ordered allocation.

It runs the same kernels as attn_sink_decode on the same inputs, only from a
different workspace, so its output must be bit-for-bit equal to
attn_sink_decode's.  Checked through the C ABI on three calls in a row: a
large workload, a smaller one, then one larger again with more splits than
the second, so that leftovers of an earlier call in the shared array,
whichever way the sizes change, would show.  One call is also compared with
the fp64 oracle.  This file is collected last on purpose."""
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


def _workload(B, Smax, Hq, Hkv, D, seed):
    g = torch.Generator().manual_seed(seed)
    seqlens = torch.randint(0, Smax + 1, (B,), generator=g, dtype=torch.int32)
    seqlens[0] = Smax
    if B > 2:
        seqlens[1] = 0
    q = torch.randn(B, Hq, D, generator=g).bfloat16()
    kc = torch.randn(B, Smax, Hkv, D, generator=g).bfloat16()
    vc = torch.randn(B, Smax, Hkv, D, generator=g).bfloat16()
    for b, n in enumerate(seqlens.tolist()):
        kc[b, n:] = float("nan")
        vc[b, n:] = float("nan")
    sinks = torch.rand(Hq, generator=g) * 12 - 4
    return q, kc, vc, seqlens, sinks


def test_noalloc_equals_decode_on_consecutive_calls():
    # (B, Smax, Hq, Hkv, D, W, seed, compare with the oracle)
    cases = [(8, 6000, 32, 4, 128, 1 << 30, 1, False),
             (5, 2500, 16, 2, 64, 700, 2, True),
             (12, 9000, 32, 4, 128, 1 << 30, 3, False)]
    for B, Smax, Hq, Hkv, D, W, seed, vs_oracle in cases:
        hq, hk, hv, hsl, hs = _workload(B, Smax, Hq, Hkv, D, seed)
        q, kc, vc, sl, sinks = (t.to(DEV) for t in (hq, hk, hv, hsl, hs))
        scale = 1.0 / np.sqrt(D)
        ref = torch.empty_like(q)
        swl.attn_sink_decode(q, kc, vc, sl, sinks, W, scale, ref)
        got = torch.full_like(q, float("nan"))
        swl.attn_sink_decode_noalloc(q, kc, vc, sl, sinks, W, scale, got)
        torch.cuda.synchronize()
        assert swl.attn_sink_get_status() == 0
        assert torch.isfinite(got.float()).all()
        assert torch.equal(got, ref), f"B={B}: differs from attn_sink_decode"
        if vs_oracle:
            want = oracle.decode(inputs.bits(hq), inputs.bits(hk), inputs.bits(hv), hsl.numpy(),
                                 hs.numpy(), W, scale)[0]
            err = float(np.abs(got.float().cpu().numpy() - want).max())
            assert err <= TOL_O, f"B={B}: max|dO| = {err} against the oracle"


def test_noalloc_rejects_workspace_beyond_the_array():
    """A workload whose workspace bound exceeds the fixed array (here 32
    splits x 128 sequences x 64 heads x 129 x 4 bytes = 135 MB) is refused
    with a clear error before anything is launched.  The cache is an
    overlapping strided view of a small buffer: the call is rejected before
    any kernel could read it."""
    B, Smax, Hq, Hkv, D = 128, 8192, 64, 8, 128
    q = torch.zeros(B, Hq, D, dtype=torch.bfloat16, device=DEV)
    base = torch.zeros(B * 8 + Smax * 8 + Hkv * 8 + D, dtype=torch.bfloat16, device=DEV)
    kc = torch.as_strided(base, (B, Smax, Hkv, D), (8, 8, 8, 1))
    sl = torch.full((B,), Smax, dtype=torch.int32, device=DEV)
    s = torch.zeros(Hq, device=DEV)
    out = torch.empty_like(q)
    with pytest.raises(RuntimeError, match="workspace"):
        swl.attn_sink_decode_noalloc(q, kc, kc, sl, s, 1 << 30, 0.088, out)
    torch.cuda.synchronize()
    assert swl.attn_sink_get_status() == 0
