"""The FMA-pipe 2^x used for part of the softmax exponentials: its coefficient
header matches its generator, and the float32 evaluation (Cody-Waite
reduction with the 1.5*2^23 shifter, degree-3 polynomial, exponent-field add)
stays within 1e-4 relative error of the exact 2^x over the range the kernel
feeds it ([-125, 8]; below that the result is a subnormal ~1e-38), well
inside bf16 rounding of P (2^-9)."""
import os
import re
import subprocess
import sys

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "sliding_window_learned_b200", "csrc")


def _coefs():
    text = open(os.path.join(CSRC, "exp2_poly.h")).read()
    return [np.float32(float(v)) for v in re.findall(r"kExp2C\d = ([-0-9.e]+)f;", text)]


def _device_steps(x):
    """The kernel's arithmetic, step by step, in float32/uint32."""
    c0, c1, c2, c3 = _coefs()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    shift = np.float32(12582912.0)
    t = (x + shift).astype(np.float32)
    nf = (t - shift).astype(np.float32)
    f = (x - nf).astype(np.float32)
    q = (f * c3 + c2).astype(np.float32)   # FMA rounding differs by at most 1 ulp per step
    q = (q * f + c1).astype(np.float32)
    q = (q * f + c0).astype(np.float32)
    bits = q.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.view(np.float32)


def test_header_matches_generator(tmp_path):
    gen = os.path.join(CSRC, "gen_exp2_poly.py")
    src = open(gen).read()
    code = src.replace("here = os.path.dirname(os.path.abspath(__file__))", f"here = {str(tmp_path)!r}")
    p = tmp_path / "gen.py"
    p.write_text(code)
    subprocess.check_call([sys.executable, str(p)], stdout=subprocess.DEVNULL)
    assert (tmp_path / "exp2_poly.h").read_text() == open(os.path.join(CSRC, "exp2_poly.h")).read()


def test_relative_error_over_kernel_range():
    x = np.concatenate([np.linspace(-125, 8, 2_000_001), np.arange(-125, 8) + 0.5,
                        np.arange(-125, 9).astype(np.float64)]).astype(np.float32)
    y = _device_steps(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1)
    assert rel.max() < 1e-4, rel.max()


def test_minus_infinity_is_negligible():
    y = _device_steps(np.array([-np.inf, -1e30, -200.0, -126.0, -125.5], np.float32))
    assert np.all(y >= 0) and np.all(y < 2.0 ** -125)
