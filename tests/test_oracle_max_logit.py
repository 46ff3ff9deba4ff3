"""Pins of the oracle's largest pre-softmax logit per (batch, head) (CPU only):
brute force over every (row, visible key) pair on small sizes, the W = 1
closed form, and the bounds the pinned forward oracle's sink-free LSE puts on
it (max_j s_ij <= LSE_i <= max_j s_ij + ln|V(i)|)."""
from __future__ import annotations

import inspect
import textwrap

import numpy as np
import pytest
import torch

import oracle
from sliding_window_learned_b200 import inputs


def _case(rng, B, L, Hq, Hkv, D):
    q = torch.from_numpy(rng.standard_normal((B, L, Hq, D)).astype(np.float32)).bfloat16()
    k = torch.from_numpy(rng.standard_normal((B, L, Hkv, D)).astype(np.float32)).bfloat16()
    return q, k


def _brute(q, k, W, scale):
    B, L, Hq, D = q.shape
    Hkv = k.shape[2]
    qd, kd = q.double().numpy(), k.double().numpy()
    out = np.full((B, Hq), -np.inf)
    for b in range(B):
        for h in range(Hq):
            hk = h // (Hq // Hkv)
            for i in range(L):
                for j in range(max(0, i - W + 1), i + 1):
                    out[b, h] = max(out[b, h], scale * float(qd[b, i, h] @ kd[b, j, hk]))
    return out


@pytest.mark.parametrize("W", [1, 2, 5, 16, 100])
def test_brute_force(W):
    rng = np.random.default_rng(W)
    q, k = _case(rng, 2, 13, 4, 2, 8)
    got = oracle.max_logit(inputs.bits(q), inputs.bits(k), W, 0.3)
    np.testing.assert_allclose(got, _brute(q, k, W, 0.3), rtol=0, atol=1e-12)


def test_window_one_closed_form():
    rng = np.random.default_rng(9)
    q, k = _case(rng, 2, 30, 6, 3, 16)
    got = oracle.max_logit(inputs.bits(q), inputs.bits(k), 1, 0.25)
    qd, kd = q.double().numpy(), k.double().numpy()
    for h in range(6):
        ref = 0.25 * np.einsum("bld,bld->bl", qd[:, :, h], kd[:, :, h // 2]).max(axis=1)
        np.testing.assert_allclose(got[:, h], ref, rtol=0, atol=1e-12)


def test_bounded_by_the_sink_free_lse():
    rng = np.random.default_rng(10)
    B, L, Hq, Hkv, D, W = 2, 40, 4, 1, 16, 7
    q, k = _case(rng, B, L, Hq, Hkv, D)
    v = torch.zeros(B, L, Hkv, D).bfloat16()
    sinks = np.full(Hq, -np.inf, np.float32)
    _, lse = oracle.fwd(inputs.bits(q), inputs.bits(k), inputs.bits(v), sinks, W, 0.5)
    got = oracle.max_logit(inputs.bits(q), inputs.bits(k), W, 0.5)
    nvis = np.minimum(np.arange(L) + 1, W)
    for b in range(B):
        for h in range(Hq):
            assert got[b, h] <= lse[b, h].max() + 1e-12
            assert got[b, h] >= (lse[b, h] - np.log(nvis)).max() - 1e-12


_MUTATIONS = {
    "window one key wider": ("for off in range(min(window, L)):", "for off in range(min(window + 1, L)):"),
    "scale not applied": ("s = float(scale) * np.einsum", "s = np.einsum"),
    "interleaved GQA": ("kh = kd[:, :, h // group, :]", "kh = kd[:, :, h % Hkv, :]"),
}


@pytest.mark.parametrize("name", sorted(_MUTATIONS))
def test_pins_reject_planted_mistake(name, monkeypatch):
    old, new = _MUTATIONS[name]
    src = textwrap.dedent(inspect.getsource(oracle.max_logit))
    assert src.count(old) == 1
    ns = dict(vars(oracle))
    exec(compile(src.replace(old, new), "<mutant>", "exec"), ns)
    monkeypatch.setattr(oracle, "max_logit", ns["max_logit"])
    with pytest.raises(AssertionError):
        for W in (1, 2, 5):
            test_brute_force(W)
        test_window_one_closed_form()
        test_bounded_by_the_sink_free_lse()
