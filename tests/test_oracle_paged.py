"""Pins of the oracle's paged-cache decode (CPU only).

The paged decode must be the contiguous decode of the cache that its block
table describes.  Each pin builds that contiguous cache independently (plain
array slicing) and compares against ``oracle.decode``, which is itself pinned
in test_oracle.py (dense sink-column softmax, split/combine exactness).
"""
from __future__ import annotations

import ctypes
import subprocess

import numpy as np
import pytest
import torch

import oracle
from sliding_window_learned_b200 import inputs


def _case(rng, B, MP, P, Hq, Hkv, D, seqlens):
    Smax = MP * P
    q = torch.from_numpy(rng.standard_normal((B, Hq, D)).astype(np.float32)).bfloat16()
    kc = torch.from_numpy(rng.standard_normal((B, Smax, Hkv, D)).astype(np.float32)).bfloat16()
    vc = torch.from_numpy(rng.standard_normal((B, Smax, Hkv, D)).astype(np.float32)).bfloat16()
    for b in range(B):
        kc[b, seqlens[b]:] = float("nan")
        vc[b, seqlens[b]:] = float("nan")
    sinks = rng.uniform(-4, 8, Hq).astype(np.float32)
    return inputs.bits(q), inputs.bits(kc), inputs.bits(vc), sinks


def _scatter(rng, kc, vc, MP, P, extra):
    """Pages of the contiguous caches placed at random physical indices of a
    pool with `extra` unused pages (NaN-filled); returns pools and table."""
    B, Smax, Hkv, D = kc.shape
    NB = B * MP + extra
    perm = rng.permutation(NB)[: B * MP].astype(np.int32)
    nan_bits = np.uint16(0x7FC0)
    kp = np.full((NB, P, Hkv, D), nan_bits, np.uint16)
    vp = np.full((NB, P, Hkv, D), nan_bits, np.uint16)
    table = perm.reshape(B, MP)
    for b in range(B):
        for p in range(MP):
            kp[table[b, p]] = kc[b, p * P:(p + 1) * P]
            vp[table[b, p]] = vc[b, p * P:(p + 1) * P]
    return kp, vp, table


@pytest.mark.parametrize("P", [1, 4, 16])
def test_identity_table_equals_contiguous(P):
    rng = np.random.default_rng(3 + P)
    B, MP, Hq, Hkv, D = 3, 48 // P, 4, 2, 8
    seqlens = np.array([0, 29, MP * P], np.int32)
    q, kc, vc, sinks = _case(rng, B, MP, P, Hq, Hkv, D, seqlens)
    kp = kc.reshape(B * MP, P, Hkv, D)
    vp = vc.reshape(B * MP, P, Hkv, D)
    table = np.arange(B * MP, dtype=np.int32).reshape(B, MP)
    for W in (1, 5, 16, 10 ** 6):
        a = oracle.decode(q, kc, vc, seqlens, sinks, W, 0.3)
        b = oracle.decode_paged(q, kp, vp, table, seqlens, sinks, W, 0.3)
        np.testing.assert_array_equal(a[0], b[0])
        np.testing.assert_array_equal(a[1], b[1])


@pytest.mark.parametrize("P", [2, 8])
def test_scattered_pages_equal_contiguous(P):
    rng = np.random.default_rng(11 + P)
    B, MP, Hq, Hkv, D = 4, 40 // P, 8, 2, 16
    seqlens = np.array([1, 17, 40, 23], np.int32)
    q, kc, vc, sinks = _case(rng, B, MP, P, Hq, Hkv, D, seqlens)
    kp, vp, table = _scatter(rng, kc, vc, MP, P, extra=5)
    for W in (1, 3, 9, 40):
        a = oracle.decode(q, kc, vc, seqlens, sinks, W, 0.25)
        b = oracle.decode_paged(q, kp, vp, table, seqlens, sinks, W, 0.25)
        np.testing.assert_array_equal(a[0], b[0])
        np.testing.assert_array_equal(a[1], b[1])


def test_shared_pages_and_out_of_range_entries():
    """Two sequences may name the same physical page (shared prefix); a table
    entry outside [0, NB) stands for a page of zero rows."""
    rng = np.random.default_rng(5)
    B, MP, P, Hq, Hkv, D = 2, 5, 4, 4, 1, 8
    seqlens = np.array([18, 20], np.int32)
    q, kc, vc, sinks = _case(rng, B, MP, P, Hq, Hkv, D, seqlens)
    kp, vp, table = _scatter(rng, kc, vc, MP, P, extra=2)
    # sequence 1 reuses sequence 0's first two pages
    table[1, :2] = table[0, :2]
    kc[1, :2 * P] = kc[0, :2 * P]
    vc[1, :2 * P] = vc[0, :2 * P]
    # page 2 of sequence 0 and page 3 of sequence 1 are out of range
    table[0, 2] = -1
    table[1, 3] = kp.shape[0]
    kc[0, 2 * P:3 * P] = 0
    vc[0, 2 * P:3 * P] = 0
    kc[1, 3 * P:4 * P] = 0
    vc[1, 3 * P:4 * P] = 0
    for W in (3, 9, 20):
        a = oracle.decode(q, kc, vc, seqlens, sinks, W, 0.5)
        b = oracle.decode_paged(q, kp, vp, table, seqlens, sinks, W, 0.5)
        np.testing.assert_array_equal(a[0], b[0])
        np.testing.assert_array_equal(a[1], b[1])


_PAGED_MUTATIONS = {
    "slot taken from the page number":
        ("int slot = t % P;", "int slot = t / P % P;"),
    "page number off by one":
        ("int32_t page = block_table[(int64_t)b * MP + t / P];",
         "int32_t page = block_table[(int64_t)b * MP + (t + 1) / P % MP];"),
    "kv head ignored in the page row":
        ("int64_t off = (((int64_t)page * P + slot) * Hkv + hk) * D;",
         "int64_t off = (((int64_t)page * P + slot) * Hkv) * D;"),
    "out-of-range entry read as page 0":
        ("memset(kd, 0, sizeof(uint16_t) * (size_t)D);",
         "memcpy(kd, kp + (int64_t)hk * D, sizeof(uint16_t) * (size_t)D);"),
    "window start off by one":
        ("int lo = n - W < 0 ? 0 : n - W;\n            for (int t = lo; t < n; ++t) {",
         "int lo = n - W + 1 < 0 ? 0 : n - W + 1;\n            for (int t = lo; t < n; ++t) {"),
}


def _pins():
    test_identity_table_equals_contiguous(4)
    test_scattered_pages_equal_contiguous(2)
    test_scattered_pages_equal_contiguous(8)
    test_shared_pages_and_out_of_range_entries()


@pytest.mark.parametrize("name", sorted(_PAGED_MUTATIONS))
def test_paged_pins_reject_planted_mistake(name, tmp_path, monkeypatch):
    old, new = _PAGED_MUTATIONS[name]
    src = open(oracle._SRC).read()
    assert src.count(old) == 1, "mutation anchor not found in oracle.c"
    path_c = tmp_path / "mutant.c"
    path_c.write_text(src.replace(old, new))
    path_so = tmp_path / "mutant.so"
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                           str(path_c), "-o", str(path_so), "-lm"])
    real = oracle._load()
    mutant = ctypes.CDLL(str(path_so))
    for fn in ("oracle_num_threads", "oracle_decode", "oracle_decode_paged"):
        getattr(mutant, fn).argtypes = getattr(real, fn).argtypes
        getattr(mutant, fn).restype = getattr(real, fn).restype
    monkeypatch.setattr(oracle, "_lib", mutant)
    with pytest.raises(AssertionError):
        _pins()
