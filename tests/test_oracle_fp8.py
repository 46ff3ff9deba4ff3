"""Pins of the oracle's FP8 (e4m3) KV-cache decode (CPU only).

- The e4m3 decoder agrees with torch's float8_e4m3fn on all 256 codes.
- With unit descales, every e4m3 value is exact in bf16, so the FP8 decode
  must equal the bf16 decode (pinned in test_oracle.py) of the same values.
- A power-of-two key descale equals the same factor folded into `scale`, and
  a power-of-two value descale scales O exactly and leaves LSE unchanged.
Planted mistakes in the FP8 code must each fail one of these."""
from __future__ import annotations

import ctypes
import subprocess

import numpy as np
import pytest
import torch

import oracle
from sliding_window_learned_b200 import inputs

NAN_CODE = 0x7F


def test_e4m3_decoder_matches_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_to_f64(int(c)) for c in range(256)])
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(got[ok], ref[ok])


def _fp8_case(rng, B, Smax, Hq, Hkv, D, seqlens):
    q = torch.from_numpy(rng.standard_normal((B, Hq, D)).astype(np.float32)).bfloat16()
    codes = rng.integers(0, 256, size=(2, B, Smax, Hkv, D)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x38          # no NaN codes inside the sequences
    # keep magnitudes moderate: exponent field <= 8 (|x| < 4)
    codes = np.where(((codes >> 3) & 15) > 8, codes & 0xC7, codes).astype(np.uint8)
    for b, n in enumerate(seqlens):
        codes[:, b, n:] = NAN_CODE                 # poison past the end
    sinks = rng.uniform(-4, 8, Hq).astype(np.float32)
    return inputs.bits(q), codes[0], codes[1], sinks


def _as_bf16_bits(codes):
    return inputs.bits(torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.bfloat16))


def test_unit_descale_equals_bf16_decode():
    rng = np.random.default_rng(4)
    B, Smax, Hq, Hkv, D = 3, 50, 8, 2, 16
    seqlens = np.array([1, 50, 23], np.int32)
    q, kc, vc, sinks = _fp8_case(rng, B, Smax, Hq, Hkv, D, seqlens)
    one = np.ones(Hkv, np.float32)
    for W in (1, 7, 50):
        a = oracle.decode_fp8(q, kc, vc, one, one, seqlens, sinks, W, 0.25)
        b = oracle.decode(q, _as_bf16_bits(kc), _as_bf16_bits(vc), seqlens, sinks, W, 0.25)
        np.testing.assert_allclose(a[0], b[0], rtol=0, atol=1e-15)
        np.testing.assert_allclose(a[1], b[1], rtol=0, atol=1e-14)


def test_descales_fold_into_scale_and_output():
    rng = np.random.default_rng(5)
    B, Smax, Hq, Hkv, D = 2, 40, 4, 2, 8
    seqlens = np.array([40, 13], np.int32)
    q, kc, vc, sinks = _fp8_case(rng, B, Smax, Hq, Hkv, D, seqlens)
    one = np.ones(Hkv, np.float32)
    base_o, base_l = oracle.decode_fp8(q, kc, vc, one, one, seqlens, sinks, 9, 0.25)
    # key descale 0.5 on every head == scale * 0.5
    o, l = oracle.decode_fp8(q, kc, vc, one * 0.5, one, seqlens, sinks, 9, 0.25)
    ref_o, ref_l = oracle.decode_fp8(q, kc, vc, one, one, seqlens, sinks, 9, 0.125)
    np.testing.assert_allclose(o, ref_o, rtol=0, atol=1e-15)
    np.testing.assert_allclose(l, ref_l, rtol=0, atol=1e-14)
    # value descale 4 on kv head 1 only: its query heads' O is 4x, the rest unchanged
    vd = np.array([1.0, 4.0], np.float32)
    o, l = oracle.decode_fp8(q, kc, vc, one, vd, seqlens, sinks, 9, 0.25)
    G = Hq // Hkv
    np.testing.assert_allclose(o[:, :G], base_o[:, :G], rtol=0, atol=0)
    np.testing.assert_allclose(o[:, G:], 4.0 * base_o[:, G:], rtol=0, atol=0)
    np.testing.assert_array_equal(l, base_l)


_FP8_MUTATIONS = {
    "exponent bias 8": ("else v = ldexp(1.0 + m / 8.0, e - 7);", "else v = ldexp(1.0 + m / 8.0, e - 8);"),
    "subnormals read as normals": ("if (e == 0) v = ldexp((double)m, -9);", "if (e == 0) v = ldexp(1.0 + m / 8.0, -6);"),
    "value descale not applied": ("o[d] += p * (vs * e4m3_to_f64(vr[d]));", "o[d] += p * e4m3_to_f64(vr[d]);"),
    "key descale taken from the value scales":
        ("double ks = (double)k_descale[hk], vs = (double)v_descale[hk];",
         "double ks = (double)v_descale[hk], vs = (double)v_descale[hk];"),
}


def _pins():
    test_e4m3_decoder_matches_torch()
    test_unit_descale_equals_bf16_decode()
    test_descales_fold_into_scale_and_output()


@pytest.mark.parametrize("name", sorted(_FP8_MUTATIONS))
def test_fp8_pins_reject_planted_mistake(name, tmp_path, monkeypatch):
    old, new = _FP8_MUTATIONS[name]
    src = open(oracle._SRC).read()
    assert src.count(old) == 1, "mutation anchor not found in oracle.c"
    path_c = tmp_path / "mutant.c"
    path_c.write_text(src.replace(old, new))
    path_so = tmp_path / "mutant.so"
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                           str(path_c), "-o", str(path_so), "-lm"])
    real = oracle._load()
    mutant = ctypes.CDLL(str(path_so))
    for fn in ("oracle_num_threads", "oracle_decode", "oracle_decode_fp8", "oracle_e4m3_to_f64"):
        getattr(mutant, fn).argtypes = getattr(real, fn).argtypes
        getattr(mutant, fn).restype = getattr(real, fn).restype
    monkeypatch.setattr(oracle, "_lib", mutant)
    with pytest.raises(AssertionError):
        _pins()
