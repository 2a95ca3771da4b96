"""Pins of the oracle's prefill gradients (CPU, float64).

``oracle.prefill_grads`` differentiates the explicit definition with torch
autograd.  These tests tie it to things other than itself: central finite
differences of the numpy forward oracle (pinned in test_oracle_pins.py), the
closed form d(rho) = -Sigma_KV dout, softmax attention's own gradients at
rho = 0, a single key, and grouped KV heads.  Planted mistakes in the torch
forward must fail the finite-difference pin.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import parallax_oracle as po

RNG = np.random.default_rng(424242)


def _case(B=1, H=2, Hkv=1, T=5, d=3, rng=RNG, rho_scale=1.0):
    q = rng.standard_normal((B, H, T, d))
    rho = rho_scale * rng.standard_normal((B, H, T, d))
    k = rng.standard_normal((B, Hkv, T, d))
    v = rng.standard_normal((B, Hkv, T, d))
    g = rng.standard_normal((B, H, T, d))
    return q, rho, k, v, g


def _loss(q, rho, k, v, g, scale, causal):
    B, H, T, _ = q.shape
    rows = [(b, h, t) for b in range(B) for h in range(H) for t in range(T)]
    out = oracle.prefill_rows(q, rho, k, v, rows, scale, causal=causal)
    return float(np.sum(out * np.stack([g[b, h, t] for b, h, t in rows])))


def _check_finite_differences(causal=True, eps=1e-6):
    q, rho, k, v, g = _case()
    grads = oracle.prefill_grads(q, rho, k, v, g, 0.7, causal=causal)
    for x, gx in zip((q, rho, k, v), grads):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            old = x[idx]
            x[idx] = old + eps
            up = _loss(q, rho, k, v, g, 0.7, causal)
            x[idx] = old - eps
            dn = _loss(q, rho, k, v, g, 0.7, causal)
            x[idx] = old
            num[idx] = (up - dn) / (2 * eps)
        np.testing.assert_allclose(gx, num, rtol=1e-6, atol=1e-7)


@pytest.mark.parametrize("causal", [True, False])
def test_grads_match_central_finite_differences(causal):
    _check_finite_differences(causal)


def test_probe_gradient_is_minus_sigma_times_dout():
    # out = vbar - Sigma^T rho, so d(dout . out)/d(rho) = -Sigma dout (Sigma is d_k x d_v).
    q, rho, k, v, g = _case(T=7, d=4)
    _, drho, _, _ = oracle.prefill_grads(q, rho, k, v, g, 0.5, causal=True)
    for h in range(2):
        for t in range(7):
            w = po.softmax_weights(0.5 * k[0, 0, :t + 1] @ q[0, h, t])
            sigma = po.sigma_kv(w, k[0, 0, :t + 1], v[0, 0, :t + 1])
            np.testing.assert_allclose(drho[0, h, t], -sigma @ g[0, h, t], rtol=1e-10, atol=1e-12)


def test_zero_probe_gives_softmax_attention_gradients():
    q, rho, k, v, g = _case(T=9, d=5)
    rho[:] = 0.0
    dq, _, dk, dv = oracle.prefill_grads(q, rho, k, v, g, 0.4, causal=True)
    Q, K, V = (torch.tensor(x, requires_grad=True) for x in (q, np.repeat(k, 2, 1), np.repeat(v, 2, 1)))
    out = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=True, scale=0.4)
    (out * torch.tensor(g)).sum().backward()
    np.testing.assert_allclose(dq, Q.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk[:, 0], K.grad.numpy().sum(1), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv[:, 0], V.grad.numpy().sum(1), rtol=1e-10, atol=1e-12)


def test_single_key_passes_dout_to_its_value_only():
    q, rho, k, v, g = _case(T=1, d=4)
    dq, drho, dk, dv = oracle.prefill_grads(q, rho, k, v, g, 0.5, causal=True)
    np.testing.assert_array_equal(dq, 0.0)
    np.testing.assert_array_equal(drho, 0.0)
    np.testing.assert_allclose(dk, 0.0, atol=1e-15)
    np.testing.assert_allclose(dv[:, 0], g.sum(1), rtol=1e-14)


def test_grouped_kv_heads_sum_their_queries_gradients():
    q, rho, k, v, g = _case(H=4, Hkv=2, T=6, d=3)
    grads = oracle.prefill_grads(q, rho, k, v, g, 0.6, causal=True)
    rep = oracle.prefill_grads(q, rho, np.repeat(k, 2, 1), np.repeat(v, 2, 1), g, 0.6, causal=True)
    np.testing.assert_allclose(grads[0], rep[0], rtol=1e-12)
    np.testing.assert_allclose(grads[1], rep[1], rtol=1e-12)
    for i in (2, 3):
        np.testing.assert_allclose(grads[i], rep[i].reshape(1, 2, 2, 6, 3).sum(2), rtol=1e-12)


def test_row_gradients_sum_to_the_prefill_gradients():
    q, rho, k, v, g = _case(H=2, Hkv=1, T=6, d=4)
    dq, drho, dk, dv = oracle.prefill_grads(q, rho, k, v, g, 0.5, causal=True)
    sk, sv = np.zeros_like(dk), np.zeros_like(dv)
    for h in range(2):
        for t in range(6):
            rq, rr, rk, rv = oracle.query_grads(q[0, h, t], rho[0, h, t], k[0, 0, :t + 1], v[0, 0, :t + 1],
                                                g[0, h, t], 0.5)
            np.testing.assert_allclose(rq, dq[0, h, t], rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(rr, drho[0, h, t], rtol=1e-12, atol=1e-14)
            sk[0, 0, :t + 1] += rk
            sv[0, 0, :t + 1] += rv
    np.testing.assert_allclose(sk, dk, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(sv, dv, rtol=1e-12, atol=1e-14)


def _mutant_transposed(Q, R, K, V, scale, causal):
    T = Q.shape[0]
    s = scale * Q @ K.T
    if causal:
        s = s.masked_fill(torch.triu(torch.ones(T, T, dtype=torch.bool), diagonal=1), float("-inf"))
    w = torch.softmax(s, dim=-1)
    vbar, kbar = w @ V, w @ K
    sigma = torch.einsum("ti,tid,tie->tde", w, K[None] - kbar[:, None], V[None] - vbar[:, None])
    return vbar - torch.einsum("tde,te->td", sigma, R)          # contracts the value side


def _mutant_weights_not_renormalised(Q, R, K, V, scale, causal):
    T = Q.shape[0]
    s = scale * Q @ K.T
    if causal:
        s = s.masked_fill(torch.triu(torch.ones(T, T, dtype=torch.bool), diagonal=1), float("-inf"))
    w = torch.exp(s - s.max(dim=-1, keepdim=True).values.detach())
    vbar, kbar = w @ V, w @ K
    sigma = torch.einsum("ti,tid,tie->tde", w, K[None] - kbar[:, None], V[None] - vbar[:, None])
    return vbar - torch.einsum("tde,td->te", sigma, R)


@pytest.mark.parametrize("mutant", [_mutant_transposed, _mutant_weights_not_renormalised])
def test_finite_difference_pin_catches_planted_mistakes(mutant, monkeypatch):
    monkeypatch.setattr(po, "_prefill_out_torch", mutant)
    with pytest.raises(AssertionError):
        _check_finite_differences(True)
