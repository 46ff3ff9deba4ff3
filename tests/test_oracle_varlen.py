"""Pins of the oracle's packed variable-length prefill (CPU only).

Each sequence of the packed layout must be attended on its own.  The pins
compare against the batched ``oracle.fwd`` (pinned in test_oracle.py) run on
an independently built padded batch: equal lengths must agree bit for bit
with a plain reshape, and unequal lengths must agree with the padded batch on
every valid row (causality means a valid query never sees the padding, which
is NaN here so that any leak shows)."""
from __future__ import annotations

import inspect
import textwrap

import numpy as np
import pytest
import torch

import oracle
from sliding_window_learned_b200 import inputs


def _packed(rng, lens, Hq, Hkv, D):
    T = int(sum(lens))
    q = torch.from_numpy(rng.standard_normal((T, Hq, D)).astype(np.float32)).bfloat16()
    k = torch.from_numpy(rng.standard_normal((T, Hkv, D)).astype(np.float32)).bfloat16()
    v = torch.from_numpy(rng.standard_normal((T, Hkv, D)).astype(np.float32)).bfloat16()
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    sinks = rng.uniform(-4, 8, Hq).astype(np.float32)
    return q, k, v, cu, sinks


def _padded(q, k, v, cu, Lmax):
    B = len(cu) - 1
    nan = float("nan")
    qp = torch.zeros((B, Lmax) + tuple(q.shape[1:]), dtype=torch.bfloat16)
    kp = torch.full((B, Lmax) + tuple(k.shape[1:]), nan, dtype=torch.bfloat16)
    vp = torch.full((B, Lmax) + tuple(v.shape[1:]), nan, dtype=torch.bfloat16)
    for b in range(B):
        n = int(cu[b + 1] - cu[b])
        qp[b, :n], kp[b, :n], vp[b, :n] = q[cu[b]:cu[b + 1]], k[cu[b]:cu[b + 1]], v[cu[b]:cu[b + 1]]
    return qp, kp, vp


def test_equal_lengths_equal_the_batched_forward():
    rng = np.random.default_rng(1)
    B, L, Hq, Hkv, D = 3, 20, 4, 2, 8
    q, k, v, cu, sinks = _packed(rng, [L] * B, Hq, Hkv, D)
    for W in (1, 7, 100):
        o, l = oracle.fwd_varlen(inputs.bits(q), inputs.bits(k), inputs.bits(v), cu, sinks, W, 0.3)
        ob, lb = oracle.fwd(inputs.bits(q.reshape(B, L, Hq, D)), inputs.bits(k.reshape(B, L, Hkv, D)),
                            inputs.bits(v.reshape(B, L, Hkv, D)), sinks, W, 0.3)
        np.testing.assert_array_equal(o, ob.reshape(B * L, Hq, D))
        np.testing.assert_array_equal(l, lb.transpose(1, 0, 2).reshape(Hq, B * L))


def test_unequal_lengths_equal_the_padded_batch():
    rng = np.random.default_rng(2)
    lens = [5, 0, 17, 1, 12]
    Hq, Hkv, D = 4, 1, 8
    q, k, v, cu, sinks = _packed(rng, lens, Hq, Hkv, D)
    qp, kp, vp = _padded(q, k, v, cu, max(lens))
    for W in (1, 4, 50):
        o, l = oracle.fwd_varlen(inputs.bits(q), inputs.bits(k), inputs.bits(v), cu, sinks, W, 0.4)
        ob, lb = oracle.fwd(inputs.bits(qp), inputs.bits(kp), inputs.bits(vp), sinks, W, 0.4)
        for b, n in enumerate(lens):
            np.testing.assert_array_equal(o[cu[b]:cu[b + 1]], ob[b, :n])
            np.testing.assert_array_equal(l[:, cu[b]:cu[b + 1]], lb[b, :, :n])


_MUTATIONS = {
    "sequence start off by one": ("s0, s1 = int(cu[b]), int(cu[b + 1])",
                                  "s0, s1 = int(cu[b]) + (1 if b else 0), int(cu[b + 1])"),
    "sequences attend across boundaries": ("o_b, l_b = fwd(q[None, s0:s1], k[None, s0:s1], v[None, s0:s1], sinks, window, scale)",
                                           "o_b, l_b = fwd(q[None, :s1], k[None, :s1], v[None, :s1], sinks, window, scale)\n        o_b, l_b = o_b[:, s0:], l_b[:, :, s0:]"),
}


@pytest.mark.parametrize("name", sorted(_MUTATIONS))
def test_varlen_pins_reject_planted_mistake(name, monkeypatch):
    old, new = _MUTATIONS[name]
    src = textwrap.dedent(inspect.getsource(oracle.fwd_varlen))
    assert src.count(old) == 1
    ns = dict(vars(oracle))
    exec(compile(src.replace(old, new), "<mutant>", "exec"), ns)
    monkeypatch.setattr(oracle, "fwd_varlen", ns["fwd_varlen"])
    with pytest.raises(AssertionError):
        test_equal_lengths_equal_the_batched_forward()
        test_unequal_lengths_equal_the_padded_batch()
