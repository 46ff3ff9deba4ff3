"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic, so both the CUDA path and the CPU oracle can be fed from
it without sharing any of the method's code.

Every workload follows one recipe: a ``torch.Generator`` on the target device,
seeded once, draws float32 values in the order q, k, v, sinks (and seqlens for
decode), and each bf16 tensor is the round-to-nearest-even cast of its float32
draw.  The oracle reads the bf16 bit patterns (``bits()``), so both sides see
identical inputs.  On a CUDA device the same recipe runs on the device's own
generator (used for the decode workload, whose KV cache is ~17 GB).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Prefill:
    """A prefill workload: Q [B,L,Hq,D], K/V [B,L,Hkv,D], sinks [Hq]."""
    name: str
    B: int
    L: int
    Hq: int
    Hkv: int
    D: int
    W: int
    sinks: tuple  # ("uniform", lo, hi) | ("normal", mean, std) | ("split", first, rest) | ("const", x)
    qk_offset: float = 0.0  # q = z1 + c, k = z2 - c (sink-dominance stress)

    @property
    def scale(self) -> float:
        return float(np.float32(1.0 / math.sqrt(self.D)))


@dataclass(frozen=True)
class Decode:
    """A single-token decode workload over a contiguous KV cache
    [B,Smax,Hkv,D] with per-sequence lengths drawn from U[n_lo, n_hi]."""
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    Smax: int
    n_lo: int
    n_hi: int
    W: int
    sinks: tuple = ("uniform", -4.0, 8.0)

    @property
    def scale(self) -> float:
        return float(np.float32(1.0 / math.sqrt(self.D)))


# The five workloads the path is specified on.
TINY = Prefill("tiny prefill B1 Hq4 Hkv2 L256 D64 W64", 1, 256, 4, 2, 64, 64,
               ("uniform", -4.0, 8.0))
PREFILL = Prefill("prefill B2 Hq32 Hkv4 L4096 D128 W513", 2, 4096, 32, 4, 128, 513,
                  ("uniform", -4.0, 8.0))
LONG_CAUSAL = Prefill("long causal B1 Hq32 Hkv8 L16384 D128 W=L", 1, 16384, 32, 8, 128,
                      16384, ("normal", 0.0, 2.0))
DECODE = Decode("split-KV decode B64 Hq32 Hkv4 D128 n~U[4096,131072]", 64, 32, 4, 128,
                131072, 4096, 131072, 131072)
# Two more decode shapes, for the bf16 and FP8 caches side by side: 16 query
# heads per kv head (two 8-head tiles per kv head), and head dim 256.
DECODE_G16 = Decode("decode G16 B64 Hq64 Hkv4 D128 n~U[4096,131072]", 64, 64, 4, 128,
                    131072, 4096, 131072, 131072)
DECODE_D256 = Decode("decode D256 B32 Hq32 Hkv4 D256 n~U[4096,131072]", 32, 32, 4, 256,
                     131072, 4096, 131072, 131072)
# Content logits near -150: q = z1 + c, k = z2 - c with c = sqrt(150 / (D*scale)).
STRESS = Prefill("sink stress B1 Hq16 Hkv2 L8192 D256 W513", 1, 8192, 16, 2, 256, 513,
                 ("split", 20.0, -50.0), qk_offset=math.sqrt(150.0 / (256 * (1 / 16))))


def _draw_sinks(spec: tuple, Hq: int, g: torch.Generator, device) -> torch.Tensor:
    kind = spec[0]
    if kind == "uniform":
        lo, hi = spec[1], spec[2]
        return torch.rand(Hq, generator=g, device=device, dtype=torch.float32) * (hi - lo) + lo
    if kind == "normal":
        return torch.randn(Hq, generator=g, device=device, dtype=torch.float32) * spec[2] + spec[1]
    if kind == "split":  # first half of the heads get spec[1], the rest spec[2]
        s = torch.full((Hq,), float(spec[2]), dtype=torch.float32, device=device)
        s[: Hq // 2] = float(spec[1])
        return s
    if kind == "const":
        return torch.full((Hq,), float(spec[1]), dtype=torch.float32, device=device)
    raise ValueError(f"unknown sink distribution {spec!r}")


def make_prefill(cfg: Prefill, seed: int = 0, device="cpu") -> dict:
    """Draw q, k, v, sinks for a prefill workload in that order."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    B, L, Hq, Hkv, D = cfg.B, cfg.L, cfg.Hq, cfg.Hkv, cfg.D
    q = torch.randn(B, L, Hq, D, generator=g, device=device, dtype=torch.float32)
    k = torch.randn(B, L, Hkv, D, generator=g, device=device, dtype=torch.float32)
    v = torch.randn(B, L, Hkv, D, generator=g, device=device, dtype=torch.float32)
    if cfg.qk_offset:
        q += cfg.qk_offset
        k -= cfg.qk_offset
    sinks = _draw_sinks(cfg.sinks, Hq, g, device)
    return dict(q=q.to(torch.bfloat16), k=k.to(torch.bfloat16), v=v.to(torch.bfloat16),
                sinks=sinks, window=cfg.W, scale=cfg.scale)


def make_decode(cfg: Decode, seed: int = 0, device="cpu", poison=True) -> dict:
    """Draw q, the KV caches, sinks and seqlens for a decode workload.

    Only the first seqlens[b] positions of each cache row are drawn; every
    later slot is set to bf16 NaN (``poison``) so that any read past a
    sequence's end shows up in the output.  The lengths are drawn first on a
    CPU generator so that they do not depend on the device."""
    gl = torch.Generator(device="cpu")
    gl.manual_seed(seed + 1)
    seqlens = torch.randint(cfg.n_lo, cfg.n_hi + 1, (cfg.B,), generator=gl, dtype=torch.int64)
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    B, Hq, Hkv, D, S = cfg.B, cfg.Hq, cfg.Hkv, cfg.D, cfg.Smax
    q = torch.randn(B, Hq, D, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    fill = float("nan") if poison else 0.0
    kc = torch.full((B, S, Hkv, D), fill, dtype=torch.bfloat16, device=device)
    vc = torch.full((B, S, Hkv, D), fill, dtype=torch.bfloat16, device=device)
    for b in range(B):
        n = int(seqlens[b])
        kc[b, :n] = torch.randn(n, Hkv, D, generator=g, device=device, dtype=torch.float32)
    for b in range(B):
        n = int(seqlens[b])
        vc[b, :n] = torch.randn(n, Hkv, D, generator=g, device=device, dtype=torch.float32)
    sinks = _draw_sinks(cfg.sinks, Hq, g, device)
    return dict(q=q, kcache=kc, vcache=vc, sinks=sinks,
                seqlens=seqlens.to(torch.int32).to(device), window=cfg.W, scale=cfg.scale)


def bits(t: torch.Tensor) -> np.ndarray:
    """The bf16 bit patterns of a tensor, as a host uint16 array."""
    assert t.dtype == torch.bfloat16
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().contiguous().cpu().numpy()
