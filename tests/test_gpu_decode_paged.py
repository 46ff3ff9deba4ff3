"""GPU parity of the paged-cache split-KV decode against the fp64 oracle.

The pools hold each sequence's pages at random physical indices; unused pages
and every cache row at a position >= seqlens[b] are bf16 NaN, and table
entries of pages that hold no visible position point at NaN pages or lie
outside the pool, so a read that should be masked shows up as NaN.  Bar (the
decode's): max|dO| <= 2e-2 and no NaN/Inf."""
import numpy as np
import pytest
import torch

import oracle
import sliding_window_learned_b200 as swl
from sliding_window_learned_b200 import inputs

pytestmark = pytest.mark.gpu
TOL_O = 2e-2
DEV = "cuda"
NAN = float("nan")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sliding_window_learned_b200 import build
    build.build()
    oracle.build()


def _paged_case(B, MP, P, Hq, Hkv, D, W, seqlens, extra, seed):
    """Contiguous caches, then the same rows scattered into NaN pools."""
    g = torch.Generator().manual_seed(seed)
    rng = np.random.default_rng(seed)
    Smax = MP * P
    q = torch.randn(B, Hq, D, generator=g).bfloat16()
    kc = torch.randn(B, Smax, Hkv, D, generator=g).bfloat16()
    vc = torch.randn(B, Smax, Hkv, D, generator=g).bfloat16()
    for b, n in enumerate(seqlens):
        kc[b, n:] = NAN
        vc[b, n:] = NAN
    sinks = torch.rand(Hq, generator=g) * 12.0 - 4.0
    NB = B * MP + extra
    perm = torch.from_numpy(rng.permutation(NB)[: B * MP].astype(np.int64))
    kp = torch.full((NB, P, Hkv, D), NAN, dtype=torch.bfloat16)
    vp = torch.full((NB, P, Hkv, D), NAN, dtype=torch.bfloat16)
    kp[perm] = kc.reshape(B * MP, P, Hkv, D)
    vp[perm] = vc.reshape(B * MP, P, Hkv, D)
    table = perm.reshape(B, MP).to(torch.int32)
    nan_page = int(np.setdiff1d(np.arange(NB), perm.numpy())[0]) if extra else -1
    for b, n in enumerate(seqlens):
        lo = max(0, n - W)
        used_hi = (n + P - 1) // P
        for pg in range(MP):
            before = (pg + 1) * P <= lo        # no visible position in this page
            after = pg >= used_hi
            if before or after:
                table[b, pg] = [nan_page, -1, NB + 7][(b + pg) % 3]
    return q, kp, vp, table, torch.tensor(seqlens, dtype=torch.int32), sinks


def _oracle(q, kp, vp, table, sl, s, W, scale):
    return oracle.decode_paged(inputs.bits(q), inputs.bits(kp), inputs.bits(vp), table.numpy(),
                               sl.numpy(), s.numpy(), W, scale)[0]


def _gpu(q, kp, vp, table, sl, s, W, scale):
    out = torch.full((q.shape[0] + 2,) + tuple(q.shape[1:]), NAN, dtype=torch.bfloat16, device=DEV)
    o = out[1:-1]
    swl.attn_sink_decode_paged(q.to(DEV), kp.to(DEV), vp.to(DEV), table.to(DEV), sl.to(DEV),
                               s.to(DEV), W, scale, o)
    torch.cuda.synchronize()
    assert swl.attn_sink_get_status() == 0
    assert bool(torch.isnan(out[0]).all()) and bool(torch.isnan(out[-1]).all()), "guard written"
    return o.float().cpu().numpy()


def _check(o, ref, what):
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    err = float(np.abs(o - ref).max())
    assert err <= TOL_O, f"{what}: max|dO| = {err}"


CASES = [  # B, MP, P, Hq, Hkv, D, W, seqlens, extra pages
    (4, 20, 16, 8, 2, 128, 1 << 30, [1, 63, 64, 320], 3),
    (3, 10, 32, 8, 1, 128, 100, [0, 320, 171], 2),
    (4, 5, 64, 32, 4, 128, 77, [320, 1, 2, 129], 4),
    (3, 4, 128, 16, 2, 64, 1, [512, 37, 128], 1),
    (2, 3, 256, 16, 1, 128, 513, [768, 600], 2),
    (3, 6, 64, 8, 2, 256, 1 << 30, [384, 100, 0], 2),
    (2, 12, 64, 6, 2, 256, 200, [700, 65], 5),
    (2, 2, 1024, 8, 2, 64, 513, [2048, 1500], 1),
    # pages smaller than a tile at the other head dims and at 16 heads per kv head
    (2, 24, 16, 8, 2, 64, 300, [380, 45], 2),
    (2, 10, 32, 4, 1, 256, 1 << 30, [300, 17], 2),
    (2, 16, 16, 32, 2, 128, 200, [250, 64], 2),
]


@pytest.mark.parametrize("case", CASES,
                         ids=[f"B{c[0]}MP{c[1]}P{c[2]}Hq{c[3]}Hkv{c[4]}D{c[5]}W{c[6]}" for c in CASES])
def test_paged_decode_against_oracle(case):
    B, MP, P, Hq, Hkv, D, W, sl, extra = case
    q, kp, vp, table, sl_t, s = _paged_case(B, MP, P, Hq, Hkv, D, W, sl, extra, seed=P + D + W % 97)
    scale = 1.0 / np.sqrt(D)
    ref = _oracle(q, kp, vp, table, sl_t, s, W, scale)
    o = _gpu(q, kp, vp, table, sl_t, s, W, scale)
    _check(o, ref, "paged decode")


def test_paged_equals_contiguous_on_the_same_rows():
    """The paged decode and the contiguous decode of the same rows agree
    (both within the oracle bar; here directly with each other)."""
    B, MP, P, Hq, Hkv, D, W = 3, 8, 64, 8, 2, 128, 300
    sl = [512, 333, 65]
    q, kp, vp, table, sl_t, s = _paged_case(B, MP, P, Hq, Hkv, D, W, sl, 2, seed=9)
    kc = torch.full((B, MP * P, Hkv, D), NAN, dtype=torch.bfloat16)
    vc = torch.full((B, MP * P, Hkv, D), NAN, dtype=torch.bfloat16)
    for b, n in enumerate(sl):
        for pg in range((n + P - 1) // P):
            idx = int(table[b, pg])
            if 0 <= idx < kp.shape[0]:        # else: a page of zero rows
                kc[b, pg * P:(pg + 1) * P] = kp[idx]
                vc[b, pg * P:(pg + 1) * P] = vp[idx]
            else:
                kc[b, pg * P:(pg + 1) * P] = 0
                vc[b, pg * P:(pg + 1) * P] = 0
        kc[b, n:] = NAN
        vc[b, n:] = NAN
    scale = 1.0 / np.sqrt(D)
    o_paged = _gpu(q, kp, vp, table, sl_t, s, W, scale)
    o_cont = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=DEV)
    swl.attn_sink_decode(q.to(DEV), kc.to(DEV), vc.to(DEV), sl_t.to(DEV), s.to(DEV), W, scale, o_cont)
    torch.cuda.synchronize()
    err = float(np.abs(o_paged - o_cont.float().cpu().numpy()).max())
    assert err <= TOL_O, err


def test_paged_decode_workload_full():
    """The decode workload (B64 Hq32 Hkv4 D128, lengths ~ U[4096, 131072])
    with its cache in 256-position pages at random pool positions: every
    output finite, and all 64 sequences against the oracle (one at a time,
    gathered from the pool by the block table on the device)."""
    cfg = inputs.DECODE
    P = 256
    y = inputs.make_decode(cfg, seed=0, device=DEV)
    B, MP = cfg.B, cfg.Smax // P
    gen = torch.Generator(device=DEV).manual_seed(1)
    perm = torch.randperm(B * MP, generator=gen, device=DEV)
    kp = torch.empty((B * MP, P, cfg.Hkv, cfg.D), dtype=torch.bfloat16, device=DEV)
    kp[perm] = y["kcache"].reshape(B * MP, P, cfg.Hkv, cfg.D)
    del y["kcache"]
    vp = torch.empty_like(kp)
    vp[perm] = y["vcache"].reshape(B * MP, P, cfg.Hkv, cfg.D)
    del y["vcache"]
    table = perm.reshape(B, MP).to(torch.int32)
    out = torch.empty_like(y["q"])
    swl.attn_sink_decode_paged(y["q"], kp, vp, table, y["seqlens"], y["sinks"], cfg.W, cfg.scale, out)
    torch.cuda.synchronize()
    assert swl.attn_sink_get_status() == 0
    o = out.float().cpu().numpy()
    assert np.isfinite(o).all()
    sl = y["seqlens"].cpu().numpy()
    tab = table.cpu()
    for b in range(B):
        n = int(sl[b])
        npg = (n + P - 1) // P
        rows = tab[b, :npg].to(DEV).long()
        kb = kp[rows].reshape(1, npg * P, cfg.Hkv, cfg.D)[:, :n]
        vb = vp[rows].reshape(1, npg * P, cfg.Hkv, cfg.D)[:, :n]
        ref = oracle.decode(inputs.bits(y["q"][b:b + 1]), inputs.bits(kb), inputs.bits(vb),
                            np.array([n], np.int32), y["sinks"].cpu().numpy(), cfg.W, cfg.scale)[0]
        _check(o[b:b + 1], ref, f"paged decode seq {b} (n={n})")


@pytest.mark.parametrize("P", [16, 32, 64])
def test_paged_strided_pools(P):
    """K and V pages interleaved in one buffer [NB, P, 2, Hkv, D] (the pools are
    strided slices of it): the tensor maps take the caller's strides, so the
    output equals that of contiguous pools bit for bit, and the oracle's."""
    B, MP, Hq, Hkv, D, W = 2, 128 // P * 3, 8, 2, 128, 200
    q, kp, vp, table, sl, s = _paged_case(B, MP, P, Hq, Hkv, D, W, [300, 97], 2, seed=P + 5)
    scale = 1.0 / np.sqrt(D)
    buf = torch.stack([kp, vp], dim=2).to(DEV)          # [NB, P, 2, Hkv, D]
    ks, vs = buf[:, :, 0], buf[:, :, 1]
    assert ks.stride()[:3] == (P * 2 * Hkv * D, 2 * Hkv * D, D)
    out = torch.empty(B, Hq, D, dtype=torch.bfloat16, device=DEV)
    swl.attn_sink_decode_paged(q.to(DEV), ks, vs, table.to(DEV), sl.to(DEV), s.to(DEV), W, scale, out)
    torch.cuda.synchronize()
    assert swl.attn_sink_get_status() == 0
    o = out.float().cpu().numpy()
    assert np.array_equal(o, _gpu(q, kp, vp, table, sl, s, W, scale))
    _check(o, _oracle(q, kp, vp, table, sl, s, W, scale), f"strided pools P={P}")
