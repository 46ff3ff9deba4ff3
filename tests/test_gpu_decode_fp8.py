"""GPU parity of the FP8 (e4m3) KV-cache decode against the fp64 oracle.

Cache slots at positions >= seqlens[b] hold the e4m3 NaN code, so a read past
a sequence's end shows up.  Bar (the decode's): max|dO| <= 2e-2, no NaN/Inf."""
import numpy as np
import pytest
import torch

import oracle
import sliding_window_learned_b200 as swl
from sliding_window_learned_b200 import inputs

pytestmark = pytest.mark.gpu
TOL_O = 2e-2
DEV = "cuda"
NAN_CODE = 0x7F


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sliding_window_learned_b200 import build
    build.build()
    oracle.build()


def _fp8_case(B, Smax, Hq, Hkv, D, seqlens, seed):
    """Random normal K/V quantised to e4m3 with a per-kv-head scale
    (amax / 448), the e4m3 NaN code past each sequence's end."""
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, D, generator=g).bfloat16()
    k = torch.randn(B, Smax, Hkv, D, generator=g) * (1.0 + torch.arange(Hkv).float())[:, None]
    v = torch.randn(B, Smax, Hkv, D, generator=g)
    kd = (k.abs().amax(dim=(0, 1, 3)) / 448.0).float()
    vd = (v.abs().amax(dim=(0, 1, 3)) / 448.0).float()
    kc = (k / kd[None, None, :, None]).to(torch.float8_e4m3fn)
    vc = (v / vd[None, None, :, None]).to(torch.float8_e4m3fn)
    kcb, vcb = kc.view(torch.uint8), vc.view(torch.uint8)
    for b, n in enumerate(seqlens):
        kcb[b, n:] = NAN_CODE
        vcb[b, n:] = NAN_CODE
    sinks = torch.rand(Hq, generator=g) * 12.0 - 4.0
    return q, kc, vc, kd, vd, torch.tensor(seqlens, dtype=torch.int32), sinks


def _oracle(q, kc, vc, kd, vd, sl, s, W, scale):
    return oracle.decode_fp8(inputs.bits(q), kc.view(torch.uint8).numpy(), vc.view(torch.uint8).numpy(),
                             kd.numpy(), vd.numpy(), sl.numpy(), s.numpy(), W, scale)[0]


def _gpu(q, kc, vc, kd, vd, sl, s, W, scale):
    out = torch.full((q.shape[0] + 2,) + tuple(q.shape[1:]), float("nan"), dtype=torch.bfloat16,
                     device=DEV)
    o = out[1:-1]
    swl.attn_sink_decode_fp8(q.to(DEV), kc.to(DEV), vc.to(DEV), kd.to(DEV), vd.to(DEV), sl.to(DEV),
                             s.to(DEV), W, scale, o)
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
    (2, 700, 16, 1, 128, 256, [700, 300]),
    (3, 333, 8, 2, 256, 1 << 30, [333, 100, 0]),
    (2, 1024, 6, 2, 256, 513, [1024, 600]),
    # many splits and 192-key tiles of the 16-heads-per-kv-head kernel (q
    # fragments in shared memory), and of the eight-warp D = 256 kernel
    (2, 20000, 32, 2, 128, 1 << 30, [20000, 12345]),
    (2, 20000, 16, 2, 256, 4096, [20000, 7777]),
]


@pytest.mark.parametrize("case", CASES, ids=[f"B{c[0]}S{c[1]}Hq{c[2]}Hkv{c[3]}D{c[4]}W{c[5]}" for c in CASES])
def test_fp8_decode_against_oracle(case):
    B, Smax, Hq, Hkv, D, W, sl = case
    q, kc, vc, kd, vd, sl_t, s = _fp8_case(B, Smax, Hq, Hkv, D, sl, seed=Smax + D + Hq)
    scale = 1.0 / np.sqrt(D)
    ref = _oracle(q, kc, vc, kd, vd, sl_t, s, W, scale)
    o = _gpu(q, kc, vc, kd, vd, sl_t, s, W, scale)
    _check(o, ref, "fp8 decode")


def test_fp8_every_code_decodes_exactly():
    """Raw random e4m3 codes (every code but NaN, subnormals and negatives
    included) with small descales, against the oracle: checks the in-kernel
    e4m3 -> bf16 conversion on the whole code table."""
    g = torch.Generator().manual_seed(8)
    B, Smax, Hq, Hkv, D = 2, 600, 8, 2, 128
    sl = [600, 333]
    q = torch.randn(B, Hq, D, generator=g).bfloat16()
    codes = torch.randint(0, 256, (2, B, Smax, Hkv, D), generator=g, dtype=torch.int32).to(torch.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x01               # no NaN inside the sequences
    for b, n in enumerate(sl):
        codes[:, b, n:] = NAN_CODE
    kc, vc = codes[0].view(torch.float8_e4m3fn), codes[1].view(torch.float8_e4m3fn)
    kd = torch.tensor([0.004, 0.002])
    vd = torch.tensor([0.01, 0.005])
    s = torch.rand(Hq, generator=g) * 12.0 - 4.0
    sl_t = torch.tensor(sl, dtype=torch.int32)
    scale = 1.0 / np.sqrt(D)
    ref = _oracle(q, kc, vc, kd, vd, sl_t, s, 1 << 30, scale)
    o = _gpu(q, kc, vc, kd, vd, sl_t, s, 1 << 30, scale)
    _check(o, ref, "fp8 decode, raw codes")


def test_fp8_unit_descales_equal_bf16_decode():
    """With unit descales the FP8 decode equals the bf16 decode of the same
    values (every e4m3 value is a bf16 value)."""
    B, Smax, Hq, Hkv, D = 3, 400, 16, 2, 128
    sl = [400, 7, 260]
    q, kc, vc, _, _, sl_t, s = _fp8_case(B, Smax, Hq, Hkv, D, sl, seed=3)
    kc = (kc.float() * 0.01).to(torch.float8_e4m3fn)     # logits of moderate size
    vc = (vc.float() / 64.0).to(torch.float8_e4m3fn)     # outputs of moderate size (|v| <= 7)
    for t in (kc, vc):
        tb = t.view(torch.uint8)
        for b, n in enumerate(sl):
            tb[b, n:] = NAN_CODE
    one = torch.ones(Hkv)
    o8 = _gpu(q, kc, vc, one, one, sl_t, s, 1 << 30, 1.0 / np.sqrt(D))
    ob = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=DEV)
    swl.attn_sink_decode(q.to(DEV), kc.to(torch.bfloat16).to(DEV), vc.to(torch.bfloat16).to(DEV),
                         sl_t.to(DEV), s.to(DEV), 1 << 30, 1.0 / np.sqrt(D), ob)
    torch.cuda.synchronize()
    assert float(np.abs(o8 - ob.float().cpu().numpy()).max()) <= TOL_O


def test_fp8_decode_workload_full():
    """The decode workload (B64 Hq32 Hkv4 D128, lengths ~ U[4096, 131072]) with
    its cache quantised to e4m3 per kv head: every output finite, and all 64
    sequences against the oracle (one at a time, valid prefix only)."""
    cfg = inputs.DECODE
    y = inputs.make_decode(cfg, seed=0, device=DEV)
    sl = y["seqlens"]
    kd = torch.empty(cfg.Hkv, device=DEV)
    vd = torch.empty(cfg.Hkv, device=DEV)
    kc = torch.empty(y["kcache"].shape, dtype=torch.float8_e4m3fn, device=DEV)
    vc = torch.empty_like(kc)
    for hk in range(cfg.Hkv):          # per kv head, slots past each end stay NaN
        for src, dst, d in ((y["kcache"], kc, kd), (y["vcache"], vc, vd)):
            x = src[:, :, hk]
            d[hk] = torch.nan_to_num(x.float(), nan=0.0).abs().amax() / 448.0
            dst[:, :, hk] = (x.float() / d[hk]).to(torch.float8_e4m3fn)
    del y["kcache"], y["vcache"]
    out = torch.empty_like(y["q"])
    swl.attn_sink_decode_fp8(y["q"], kc, vc, kd, vd, sl, y["sinks"], cfg.W, cfg.scale, out)
    torch.cuda.synchronize()
    assert swl.attn_sink_get_status() == 0
    o = out.float().cpu().numpy()
    assert np.isfinite(o).all()
    sln = sl.cpu().numpy()
    for b in range(cfg.B):
        n = int(sln[b])
        ref = oracle.decode_fp8(inputs.bits(y["q"][b:b + 1]), kc[b:b + 1, :n].view(torch.uint8).cpu().numpy(),
                                vc[b:b + 1, :n].view(torch.uint8).cpu().numpy(), kd.cpu().numpy(),
                                vd.cpu().numpy(), np.array([n], np.int32), y["sinks"].cpu().numpy(),
                                cfg.W, cfg.scale)[0]
        _check(o[b:b + 1], ref, f"fp8 decode seq {b} (n={n})")
