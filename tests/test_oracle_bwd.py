"""Pins of the oracle's backward pass (CPU only).

- Its differentiable forward is the pinned C forward oracle (to 1e-12).
- Central finite differences of the loss sum(dO * O) along random directions
  agree with the gradients (q, k, v and the sinks).
- The sink gradient has the closed form dsink_h = -sum_i P_sink,i (dO_i . O_i)
  with P_sink,i = exp(sink_h - LSE_i), LSE from the C oracle.
- With every sink at -inf, dq/dk/dv equal torch's own fp64 backward of
  scaled_dot_product_attention with the window mask, and dsink is 0.
Planted mistakes in the backward's forward must each fail one of these."""
from __future__ import annotations

import inspect
import textwrap

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from sliding_window_learned_b200 import inputs


def _case(seed, B=2, L=9, Hq=4, Hkv=2, D=8, sinks=None):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, L, Hq, D, generator=g).bfloat16()
    k = torch.randn(B, L, Hkv, D, generator=g).bfloat16()
    v = torch.randn(B, L, Hkv, D, generator=g).bfloat16()
    do = torch.randn(B, L, Hq, D, generator=g).bfloat16()
    if sinks is None:
        sinks = (torch.rand(Hq, generator=g) * 6.0 - 2.0).numpy().astype(np.float32)
    return q, k, v, do, sinks


def test_forward_is_the_c_oracle():
    q, k, v, do, s = _case(1)
    for W in (1, 3, 100):
        *_, o, lse = oracle.bwd(inputs.bits(q), inputs.bits(k), inputs.bits(v), s, inputs.bits(do), W, 0.3)
        oc, lc = oracle.fwd(inputs.bits(q), inputs.bits(k), inputs.bits(v), s, W, 0.3)
        np.testing.assert_allclose(o, oc, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, lc, rtol=0, atol=1e-12)


def test_finite_differences():
    q, k, v, do, s = _case(2)
    W, scale = 4, 0.3
    dq, dk, dv, ds, _, _ = oracle.bwd(inputs.bits(q), inputs.bits(k), inputs.bits(v), s, inputs.bits(do),
                                      W, scale)
    x = [torch.from_numpy(oracle._bits_to_f64(inputs.bits(t))) for t in (q, k, v)]
    sd = torch.from_numpy(s.astype(np.float64))
    dod = torch.from_numpy(oracle._bits_to_f64(inputs.bits(do)))
    grads = [dq, dk, dv, ds]
    rng = np.random.default_rng(3)

    def loss(xs, ss):
        o, _ = oracle._torch_forward(xs[0], xs[1], xs[2], ss, W, scale)
        return float((o * dod).sum())

    h = 1e-5
    for which in range(4):
        base = x[which] if which < 3 else sd
        u = torch.from_numpy(rng.standard_normal(tuple(base.shape)))
        plus = [t.clone() for t in x] + [sd.clone()]
        minus = [t.clone() for t in x] + [sd.clone()]
        plus[which] = plus[which] + h * u
        minus[which] = minus[which] - h * u
        fd = (loss(plus[:3], plus[3]) - loss(minus[:3], minus[3])) / (2 * h)
        an = float((torch.from_numpy(grads[which]) * u).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (which, fd, an)


def test_sink_gradient_closed_form():
    q, k, v, do, s = _case(4, L=12)
    W, scale = 5, 0.25
    _, _, _, ds, _, _ = oracle.bwd(inputs.bits(q), inputs.bits(k), inputs.bits(v), s, inputs.bits(do),
                                   W, scale)
    oc, lc = oracle.fwd(inputs.bits(q), inputs.bits(k), inputs.bits(v), s, W, scale)
    dod = oracle._bits_to_f64(inputs.bits(do))
    Dsum = (dod * oc).sum(-1)                                   # [B, L, Hq]
    psink = np.exp(s.astype(np.float64)[None, :, None] - lc)    # [B, Hq, L]
    ref = -(psink * Dsum.transpose(0, 2, 1)).sum(axis=(0, 2))
    np.testing.assert_allclose(ds, ref, rtol=1e-12, atol=1e-12)


def test_no_sink_equals_torch_sdpa_backward():
    B, L, Hq, Hkv, D, W = 2, 11, 4, 2, 8, 3
    q, k, v, do, _ = _case(5, B, L, Hq, Hkv, D)
    s = np.full(Hq, -np.inf, np.float32)
    dq, dk, dv, ds, _, _ = oracle.bwd(inputs.bits(q), inputs.bits(k), inputs.bits(v), s, inputs.bits(do),
                                      W, 0.35)
    qt = q.double().permute(0, 2, 1, 3).requires_grad_()
    kt = k.double().repeat_interleave(Hq // Hkv, dim=2).permute(0, 2, 1, 3).detach().requires_grad_()
    vt = v.double().repeat_interleave(Hq // Hkv, dim=2).permute(0, 2, 1, 3).detach().requires_grad_()
    i = torch.arange(L).view(L, 1)
    j = torch.arange(L).view(1, L)
    mask = (j <= i) & (j >= i - W + 1)
    o = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=float(np.float32(0.35)))
    (o * do.double().permute(0, 2, 1, 3)).sum().backward()
    np.testing.assert_allclose(dq, qt.grad.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)
    dk_ref = kt.grad.permute(0, 2, 1, 3).reshape(B, L, Hkv, Hq // Hkv, D).sum(3).numpy()
    dv_ref = vt.grad.permute(0, 2, 1, 3).reshape(B, L, Hkv, Hq // Hkv, D).sum(3).numpy()
    np.testing.assert_allclose(dk, dk_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv, dv_ref, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(ds, np.zeros(Hq))


_MUTATIONS = {
    "sink left out of the softmax": (
        'full = torch.cat([s, sinks.view(1, Hq, 1, 1).expand(B, Hq, L, 1)], dim=-1)',
        'full = torch.cat([s, sinks.view(1, Hq, 1, 1).expand(B, Hq, L, 1) - 1e9], dim=-1)'),
    "window one key too wide": ('visible = (j <= i) & (j >= i - int(window) + 1)',
                                'visible = (j <= i) & (j >= i - int(window))'),
    "interleaved GQA": ('kk = kd.repeat_interleave(Hq // Hkv, dim=2)', 'kk = kd.repeat(1, 1, Hq // Hkv, 1)'),
}


@pytest.mark.parametrize("name", sorted(_MUTATIONS))
def test_pins_reject_planted_mistake(name, monkeypatch):
    old, new = _MUTATIONS[name]
    src = textwrap.dedent(inspect.getsource(oracle._torch_forward))
    assert src.count(old) == 1
    ns = dict(vars(oracle))
    exec(compile(src.replace(old, new), "<mutant>", "exec"), ns)
    monkeypatch.setattr(oracle, "_torch_forward", ns["_torch_forward"])
    with pytest.raises(AssertionError):
        test_forward_is_the_c_oracle()
        test_sink_gradient_closed_form()
        test_no_sink_equals_torch_sdpa_backward()
