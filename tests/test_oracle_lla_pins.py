"""Pins of the oracle's Local Linear Attention with the solved probe.

LLA is the local linear estimate at the query: the intercept of the
softmax-weighted least-squares fit v ~ a + M^T (k - q) (newx.sg "Abstract";
wispaper blog, "Context: Why Softmax is Not Enough").  The oracle computes it
as vbar - S_KV^T rho* with (S_KK + ridge I) rho* = kbar - q.  These tests pin
that against facts computed another way:

  * the intercept of the weighted fit from numpy's lstsq, with no ridge and
    with a ridge penalty on the slope (lstsq on the augmented system);
  * a local linear estimator reproduces affine data exactly;
  * a huge ridge leaves softmax attention (torch's SDPA);
  * a single key has a closed-form probe.
Planted mistakes (wrong sign of the right-hand side, uncentred second
moment, unnormalised weights, ridge on the intercept) must fail a pin.
"""

import math

import numpy as np
import pytest
import torch

import oracle

RNG = np.random.default_rng(20261203)


def _problem(n, d, dv=None, rng=RNG):
    q = rng.standard_normal(d)
    K = rng.standard_normal((n, d))
    V = rng.standard_normal((n, dv or d))
    return q, K, V


def _weights(q, K, scale):
    s = scale * (K @ q)
    w = np.exp(s - s.max())
    return w / w.sum()


def _ridge_wls_intercept(q, K, V, w, ridge):
    """argmin_a,M sum_i w_i |v_i - a - M^T (k_i - q)|^2 + ridge |M|_F^2 by
    lstsq on the system stacked with sqrt(ridge) I rows for the slope."""
    n, d = K.shape
    X = np.concatenate([np.ones((n, 1)), K - q], axis=1) * np.sqrt(w)[:, None]
    Y = V * np.sqrt(w)[:, None]
    if ridge > 0:
        X = np.concatenate([X, np.concatenate([np.zeros((d, 1)), math.sqrt(ridge) * np.eye(d)], axis=1)])
        Y = np.concatenate([Y, np.zeros((d, V.shape[1]))])
    coef, *_ = np.linalg.lstsq(X, Y, rcond=None)
    return coef[0]


@pytest.mark.parametrize("n,d,ridge", [(20, 4, 0.0), (300, 16, 0.0), (50, 8, 0.3), (5, 8, 0.05), (2000, 32, 1e-3)])
def test_intercept_of_the_weighted_fit(n, d, ridge):
    q, K, V = _problem(n, d, dv=d + 3)
    scale = 1.0 / math.sqrt(d)
    _, out = oracle.lla_query(q, K, V, scale, ridge)
    ref = _ridge_wls_intercept(q, K, V, _weights(q, K, scale), ridge)
    np.testing.assert_allclose(out, ref, rtol=1e-8, atol=1e-9)


@pytest.mark.parametrize("n,d", [(12, 4), (200, 16)])
def test_affine_data_is_reproduced_exactly(n, d):
    # v = a + B^T k for every key: the local linear estimate at q is a + B^T q,
    # whatever the weights (softmax attention would return a + B^T kbar).
    q, K, _ = _problem(n, d)
    a = RNG.standard_normal(5)
    Bm = RNG.standard_normal((d, 5))
    V = a + K @ Bm
    _, out = oracle.lla_query(q, K, V, 0.9, 0.0)
    np.testing.assert_allclose(out, a + Bm.T @ q, rtol=1e-9, atol=1e-9)


def test_huge_ridge_is_softmax_attention():
    q, K, V = _problem(100, 8)
    scale = 0.35
    rho, out = oracle.lla_query(q, K, V, scale, 1e12)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None, None], torch.from_numpy(K)[None, None],
        torch.from_numpy(V)[None, None], scale=scale)[0, 0, 0].numpy()
    assert np.abs(rho).max() < 1e-10
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-10)


def test_single_key_closed_form():
    # One key: S_KK = 0, so rho* = (k - q) / ridge and the output is the value.
    q, K, V = _problem(1, 6)
    rho, out = oracle.lla_query(q, K, V, 0.5, 0.25)
    np.testing.assert_allclose(rho, (K[0] - q) / 0.25, rtol=1e-14)
    np.testing.assert_allclose(out, V[0], rtol=0, atol=1e-14)


def test_empty_key_set():
    rho, out = oracle.lla_query(np.ones(4), np.zeros((0, 4)), np.zeros((0, 3)), 1.0, 0.1)
    assert not rho.any() and not out.any()


def test_decode_layouts_match_per_query_calls():
    # GQA, ragged lengths and a paged copy of the same cache give the
    # per-query answers.
    B, Hq, Hkv, d, L = 2, 4, 2, 8, 40
    q = RNG.standard_normal((B, Hq, d))
    k = RNG.standard_normal((B, Hkv, L, d))
    v = RNG.standard_normal((B, Hkv, L, d))
    lens = [40, 23]
    rho, out = oracle.lla_decode(q, k, v, 0.4, 0.1, seq_lens=lens)
    pages = np.full((2 * 1 + 2, Hkv, 32, d), np.nan)
    vpages = np.full_like(pages, np.nan)
    table = np.array([[3, 0], [1, -1]])
    for b, row in enumerate(table):
        for j, pg in enumerate(row):
            if pg >= 0:
                take = min(32, lens[b] - 32 * j)
                pages[pg, :, :take] = k[b, :, 32 * j:32 * j + take]
                vpages[pg, :, :take] = v[b, :, 32 * j:32 * j + take]
    rho_p, out_p = oracle.lla_decode(q, pages, vpages, 0.4, 0.1, seq_lens=lens, page_table=table)
    for b in range(B):
        for h in range(Hq):
            r, o = oracle.lla_query(q[b, h], k[b, h // 2, :lens[b]], v[b, h // 2, :lens[b]], 0.4, 0.1)
            np.testing.assert_allclose(rho[b, h], r, rtol=1e-12)
            np.testing.assert_allclose(out[b, h], o, rtol=1e-12)
            np.testing.assert_allclose(rho_p[b, h], r, rtol=1e-12)
            np.testing.assert_allclose(out_p[b, h], o, rtol=1e-12)


# ---------------------------------------------------------- planted mistakes


def _probe_with(q, keys, scale, ridge, *, center=True, normalise=True, rhs_sign=1.0, ridge_on="slope"):
    K = np.asarray(keys, dtype=np.float64)
    q = np.asarray(q, dtype=np.float64)
    if K.shape[0] == 0:
        return np.zeros(K.shape[1])
    s = scale * (K @ q)
    w = np.exp(s - s.max())
    if normalise:
        w = w / w.sum()
    kbar = w @ K
    Kc = K - kbar if center else K
    A = Kc.T @ (w[:, None] * Kc)
    if ridge_on == "slope":
        A = A + ridge * np.eye(K.shape[1])
    else:   # a mistake: the penalty also lands on the right-hand side
        A = A + ridge * np.eye(K.shape[1])
        kbar = kbar + ridge
    return np.linalg.solve(A, rhs_sign * (kbar - q))


MUTANTS = {
    "flipped_rhs": dict(rhs_sign=-1.0),
    "uncentred_second_moment": dict(center=False),
    "unnormalised_weights": dict(normalise=False),
    "ridge_leaks_into_rhs": dict(ridge_on="both"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistakes(name, monkeypatch):
    from oracle import parallax_oracle as po
    kw = MUTANTS[name]
    monkeypatch.setattr(po, "lla_probe", lambda q, keys, scale, ridge: _probe_with(q, keys, scale, ridge, **kw))
    failures = 0
    for pin in (lambda: test_intercept_of_the_weighted_fit(50, 8, 0.3),
                lambda: test_intercept_of_the_weighted_fit(300, 16, 0.0),
                lambda: test_affine_data_is_reproduced_exactly(12, 4),
                test_single_key_closed_form):
        try:
            pin()
        except (AssertionError, np.linalg.LinAlgError):
            failures += 1
    assert failures > 0, f"{name} passed every pin"


def test_unmutated_probe_passes_the_same_pins():
    for pin in (lambda: test_intercept_of_the_weighted_fit(50, 8, 0.3),
                lambda: test_affine_data_is_reproduced_exactly(12, 4), test_single_key_closed_form):
        pin()
