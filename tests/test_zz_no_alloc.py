"""attn_sink_decode_noalloc: the decode entry point for callers that may not
allocate device memory while decoding (engines that reserve nearly all of HBM
for their KV cache up front, or runtimes whose allocator owns every device
byte).  Its workspace is the library's fixed device array instead of a
stream-ordered allocation.

Checked through the C ABI against attn_sink_decode on the same inputs, on two
calls in a row with different workloads, so that anything the second call
wrongly inherited from the first call's leftovers in the shared array would
show.  This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import sliding_window_learned_b200 as swl

pytestmark = pytest.mark.gpu
TOL_O = 2e-2
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sliding_window_learned_b200 import build
    build.build()


def _workload(B, Smax, Hq, Hkv, D, seed):
    g = torch.Generator().manual_seed(seed)
    seqlens = torch.randint(0, Smax + 1, (B,), generator=g, dtype=torch.int32)
    seqlens[0] = Smax
    if B > 2:
        seqlens[1] = 0
    q = torch.randn(B, Hq, D, generator=g).bfloat16().to(DEV)
    kc = torch.randn(B, Smax, Hkv, D, generator=g).bfloat16().to(DEV)
    vc = torch.randn(B, Smax, Hkv, D, generator=g).bfloat16().to(DEV)
    sinks = (torch.rand(Hq, generator=g) * 12 - 4).to(DEV)
    return q, kc, vc, seqlens.to(DEV), sinks


def test_noalloc_matches_decode_on_consecutive_calls():
    cases = [(8, 6000, 32, 4, 128, 1 << 30, 1), (5, 2500, 16, 2, 64, 700, 2)]
    for B, Smax, Hq, Hkv, D, W, seed in cases:
        q, kc, vc, sl, sinks = _workload(B, Smax, Hq, Hkv, D, seed)
        scale = 1.0 / np.sqrt(D)
        ref = torch.empty_like(q)
        swl.attn_sink_decode(q, kc, vc, sl, sinks, W, scale, ref)
        got = torch.full_like(q, float("nan"))
        swl.attn_sink_decode_noalloc(q, kc, vc, sl, sinks, W, scale, got)
        torch.cuda.synchronize()
        assert swl.attn_sink_get_status() == 0
        r = ref.float().cpu().numpy()
        o = got.float().cpu().numpy()
        assert np.isfinite(o).all()
        assert float(np.abs(o - r).max()) <= TOL_O
