"""Pins of the float64 oracle to facts fixed outside the oracle itself.

Each test checks the oracle against something it does not compute the same
way: hand-worked exact examples, a library routine that the definition
reduces to, the textbook weighted-least-squares local linear estimate, a
pairwise brute-force double sum, closed forms and invariants of the
definition.  The mutation tests at the end plant plausible mistakes into the
oracle (on the CPU) and check that the pins catch them.
"""

import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import parallax_oracle as po
from tests.golden.loader import load_worked_examples

RNG = np.random.default_rng(20260527)


def _rand_problem(n, d, dv=None, rng=RNG, kscale=1.0):
    dv = dv or d
    q = rng.standard_normal(d)
    rho = rng.standard_normal(d)
    K = kscale * rng.standard_normal((n, d))
    V = rng.standard_normal((n, dv))
    return q, rho, K, V


# --------------------------------------------------------------------------
# Hand-derived worked examples (tests/golden/worked_examples.txt)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("name", sorted(load_worked_examples()))
def test_worked_examples(name):
    c = load_worked_examples()[name]
    out = oracle.parallax_query(c["q"], c["rho"], c["k"], c["v"], c["scale"])
    np.testing.assert_allclose(out, c["out"], rtol=0, atol=1e-13)


def test_worked_example_as_causal_prefill():
    # A T = 2 causal prefill over the keys of [two_keys_equal_weights]: row 0
    # sees only key 0 (output v_0); row 1 sees both (the worked answer).
    c = load_worked_examples()["two_keys_equal_weights"]
    q = np.stack([np.array([7.0, -2.0]), c["q"]])[None, None]
    rho = np.stack([np.array([1.0, 1.0]), c["rho"]])[None, None]
    k = c["k"][None, None]
    v = c["v"][None, None]
    out = oracle.prefill_rows(q, rho, k, v, [(0, 0, 0), (0, 0, 1)], c["scale"], causal=True)
    np.testing.assert_allclose(out[0], c["v"][0], atol=0)
    np.testing.assert_allclose(out[1], c["out"], atol=1e-13)


# --------------------------------------------------------------------------
# Special cases that reduce to a library routine or a textbook estimator
# --------------------------------------------------------------------------

@pytest.mark.parametrize("n,d", [(1, 4), (7, 8), (64, 16), (300, 64)])
def test_rho_zero_is_softmax_attention(n, d):
    """rho = 0 leaves the local constant (Nadaraya-Watson) estimate: plain
    softmax attention, here torch's scaled_dot_product_attention in float64."""
    q, _, K, V = _rand_problem(n, d)
    scale = 1.0 / math.sqrt(d)
    ours = oracle.parallax_query(q, np.zeros(d), K, V, scale)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None, None], torch.from_numpy(K)[None, None],
        torch.from_numpy(V)[None, None], scale=scale)[0, 0, 0].numpy()
    np.testing.assert_allclose(ours, ref, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("n,d", [(6, 2), (20, 4), (200, 8)])
def test_solved_probe_gives_local_linear_regression(n, d):
    """With the solved probe rho* = Sigma_KK^{-1} (kbar - q) (what Local Linear
    Attention obtains with a per-token solver), the output is the intercept of
    the softmax-weighted least-squares fit v ~ a + M^T (k - q), evaluated at
    the query.  The fit is done with numpy's lstsq, independent of the oracle.
    This pins the sign of the correction and that rho contracts the key side.
    """
    q, _, K, V = _rand_problem(n, d, dv=d + 1)
    scale = 0.7
    s = scale * (K @ q)
    w = np.exp(s - s.max())
    w /= w.sum()
    kbar = w @ K
    Kc = K - kbar
    S_kk = Kc.T @ (w[:, None] * Kc)
    rho_star = np.linalg.solve(S_kk, kbar - q)

    X = np.concatenate([np.ones((n, 1)), K - q], axis=1)
    sw = np.sqrt(w)[:, None]
    coef, *_ = np.linalg.lstsq(sw * X, sw * V, rcond=None)
    intercept = coef[0]

    ours = oracle.parallax_query(q, rho_star, K, V, scale)
    np.testing.assert_allclose(ours, intercept, rtol=1e-9, atol=1e-9)


# --------------------------------------------------------------------------
# Closed forms and brute force
# --------------------------------------------------------------------------

@pytest.mark.parametrize("seed", range(5))
def test_two_key_closed_form(seed):
    """Two keys: w1 = 1 / (1 + exp(-scale q.(k1 - k2))), Sigma_KV =
    w1 w2 (k1 - k2)(v1 - v2)^T, so out = w1 v1 + w2 v2 - w1 w2 (rho.dk) dv."""
    rng = np.random.default_rng(seed)
    d = 5
    q, rho, K, V = _rand_problem(2, d, rng=rng)
    scale = 0.3 + seed * 0.2
    w1 = 1.0 / (1.0 + math.exp(-scale * float(q @ (K[0] - K[1]))))
    w2 = 1.0 - w1
    expect = w1 * V[0] + w2 * V[1] - w1 * w2 * float(rho @ (K[0] - K[1])) * (V[0] - V[1])
    np.testing.assert_allclose(oracle.parallax_query(q, rho, K, V, scale), expect,
                               rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("n,d", [(1, 1), (2, 3), (3, 2), (5, 4), (8, 4), (8, 1)])
def test_pairwise_brute_force(n, d):
    """Pure-Python loops over the pairwise form of the weighted covariance,
    Sigma_KV = 1/2 sum_i sum_j w_i w_j (k_i - k_j)(v_i - v_j)^T, which needs no
    weighted means; the weights come from math.exp on each score."""
    rng = np.random.default_rng(100 * n + d)
    q, rho, K, V = _rand_problem(n, d, rng=rng)
    scale = 0.9
    s = [scale * sum(q[c] * K[i][c] for c in range(d)) for i in range(n)]
    top = max(s)
    e = [math.exp(x - top) for x in s]
    tot = sum(e)
    w = [x / tot for x in e]
    vbar = [sum(w[i] * V[i][c] for i in range(n)) for c in range(d)]
    sig = [[0.0] * d for _ in range(d)]
    for i, j in itertools.product(range(n), range(n)):
        for a in range(d):
            for b in range(d):
                sig[a][b] += 0.5 * w[i] * w[j] * (K[i][a] - K[j][a]) * (V[i][b] - V[j][b])
    expect = [vbar[b] - sum(sig[a][b] * rho[a] for a in range(d)) for b in range(d)]
    np.testing.assert_allclose(oracle.parallax_query(q, rho, K, V, scale), expect,
                               rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(oracle.sigma_kv(np.array(w), K, V), np.array(sig),
                               rtol=1e-11, atol=1e-12)


# --------------------------------------------------------------------------
# Invariants of the definition
# --------------------------------------------------------------------------

def test_single_key_and_identical_values():
    q, rho, K, V = _rand_problem(1, 6)
    np.testing.assert_array_equal(oracle.parallax_query(q, rho, K, V, 0.4), V[0])
    q, rho, K, V = _rand_problem(50, 6)
    V[:] = V[0]
    np.testing.assert_allclose(oracle.parallax_query(q, rho, K, V, 0.4), V[0], atol=1e-13)


def test_identical_keys_give_mean_of_values():
    q, rho, K, V = _rand_problem(40, 6)
    K[:] = K[3]
    np.testing.assert_allclose(oracle.parallax_query(q, rho, K, V, 0.4), V.mean(0),
                               rtol=1e-12, atol=1e-13)


def test_key_translation_invariance_and_value_equivariance():
    q, rho, K, V = _rand_problem(33, 8)
    base = oracle.parallax_query(q, rho, K, V, 0.35)
    mu = 3.0 * RNG.standard_normal(8)
    np.testing.assert_allclose(oracle.parallax_query(q, rho, K + mu, V, 0.35), base,
                               rtol=1e-9, atol=1e-10)
    b = RNG.standard_normal(8)
    np.testing.assert_allclose(oracle.parallax_query(q, rho, K, V + b, 0.35), base + b,
                               rtol=1e-12, atol=1e-12)


def test_output_is_affine_in_rho():
    q, r1, K, V = _rand_problem(25, 7)
    r2 = RNG.standard_normal(7)
    vbar = oracle.parallax_query(q, np.zeros(7), K, V, 0.5)
    f = lambda r: oracle.parallax_query(q, r, K, V, 0.5) - vbar  # noqa: E731
    np.testing.assert_allclose(f(2.0 * r1 - 3.0 * r2), 2.0 * f(r1) - 3.0 * f(r2),
                               rtol=1e-11, atol=1e-12)


def test_key_permutation_invariance():
    q, rho, K, V = _rand_problem(41, 8)
    p = RNG.permutation(41)
    np.testing.assert_allclose(oracle.parallax_query(q, rho, K[p], V[p], 0.5),
                               oracle.parallax_query(q, rho, K, V, 0.5), rtol=1e-12, atol=1e-13)


def test_empty_key_set_is_zero():
    out = oracle.parallax_query(np.ones(4), np.ones(4), np.zeros((0, 4)), np.zeros((0, 4)), 1.0)
    np.testing.assert_array_equal(out, np.zeros(4))


# --------------------------------------------------------------------------
# Layout readings: GQA, sequence lengths, paging, causal prefill
# --------------------------------------------------------------------------

def test_gqa_equals_repeated_kv_heads():
    B, Hq, Hkv, L, d = 2, 6, 2, 17, 4
    q = RNG.standard_normal((B, Hq, d))
    rho = RNG.standard_normal((B, Hq, d))
    k = RNG.standard_normal((B, Hkv, L, d))
    v = RNG.standard_normal((B, Hkv, L, d))
    gqa = oracle.decode(q, rho, k, v, 0.5)
    mha = oracle.decode(q, rho, np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1), 0.5)
    np.testing.assert_array_equal(gqa, mha)


def test_seq_lens_ignore_the_tail():
    B, H, L, d = 3, 2, 20, 4
    q = RNG.standard_normal((B, H, d))
    rho = RNG.standard_normal((B, H, d))
    k = RNG.standard_normal((B, H, L, d))
    v = RNG.standard_normal((B, H, L, d))
    lens = [20, 7, 1]
    for b, n in enumerate(lens):
        k[b, :, n:] = np.nan
        v[b, :, n:] = np.nan
    out = oracle.decode(q, rho, k, v, 0.5, seq_lens=lens)
    assert np.isfinite(out).all()
    for b, n in enumerate(lens):
        for h in range(H):
            np.testing.assert_array_equal(
                out[b, h], oracle.parallax_query(q[b, h], rho[b, h], k[b, h, :n], v[b, h, :n], 0.5))


def test_paged_gather_matches_contiguous():
    B, Hkv, g, d, ps = 3, 2, 2, 4, 8
    lens = [19, 8, 1]
    L = 24
    q = RNG.standard_normal((B, Hkv * g, d))
    rho = RNG.standard_normal((B, Hkv * g, d))
    kc = RNG.standard_normal((B, Hkv, L, d))
    vc = RNG.standard_normal((B, Hkv, L, d))
    n_pages = [-(-n // ps) for n in lens]
    perm = RNG.permutation(sum(n_pages))
    kp = np.full((sum(n_pages), Hkv, ps, d), np.nan)
    vp = np.full_like(kp, np.nan)
    table = -np.ones((B, 3), dtype=np.int64)
    nxt = 0
    for b, n in enumerate(lens):
        for j in range(n_pages[b]):
            page = perm[nxt]
            nxt += 1
            table[b, j] = page
            take = min(ps, n - j * ps)
            kp[page, :, :take] = kc[b, :, j * ps:j * ps + take]
            vp[page, :, :take] = vc[b, :, j * ps:j * ps + take]
    paged = oracle.decode(q, rho, kp, vp, 0.5, seq_lens=lens, page_table=table)
    contig = oracle.decode(q, rho, kc, vc, 0.5, seq_lens=lens)
    np.testing.assert_array_equal(paged, contig)


def test_prefill_rows_equal_decode_over_prefix():
    B, H, Hkv, T, d = 2, 4, 2, 13, 4
    q = RNG.standard_normal((B, H, T, d))
    rho = RNG.standard_normal((B, H, T, d))
    k = RNG.standard_normal((B, Hkv, T, d))
    v = RNG.standard_normal((B, Hkv, T, d))
    rows = [(b, h, t) for b in range(B) for h in range(H) for t in (0, 1, 6, T - 1)]
    out = oracle.prefill_rows(q, rho, k, v, rows, 0.5, causal=True)
    for (b, h, t), o in zip(rows, out):
        kvh = h // 2
        ref = oracle.decode(q[b, h, t][None, None], rho[b, h, t][None, None],
                            k[b, kvh, :t + 1][None, None], v[b, kvh, :t + 1][None, None], 0.5)[0, 0]
        np.testing.assert_array_equal(o, ref)
        if t == 0:
            np.testing.assert_array_equal(o, v[b, kvh, 0])
    full = oracle.prefill_rows(q, rho, k, v, [(1, 3, 2)], 0.5, causal=False)[0]
    np.testing.assert_array_equal(
        full, oracle.parallax_query(q[1, 3, 2], rho[1, 3, 2], k[1, 1], v[1, 1], 0.5))


# --------------------------------------------------------------------------
# Chunked (append) prefill over a paged cache
# --------------------------------------------------------------------------

def _to_pages(seqs, ps, rng, fill=np.nan):
    """Place per-sequence [Hkv, L_b, d] arrays into a permuted page pool."""
    Hkv, d = seqs[0].shape[0], seqs[0].shape[2]
    n_pages = [-(-s.shape[1] // ps) for s in seqs]
    perm = rng.permutation(max(1, sum(n_pages)))
    pool = np.full((max(1, sum(n_pages)), Hkv, ps, d), fill)
    table = -np.ones((len(seqs), max(1, max(n_pages))), dtype=np.int64)
    nxt = 0
    for b, s in enumerate(seqs):
        for j in range(n_pages[b]):
            page = perm[nxt]
            nxt += 1
            table[b, j] = page
            take = min(ps, s.shape[1] - j * ps)
            pool[page, :, :take] = s[:, j * ps:j * ps + take]
    return pool, table


def _chunked_case(rng):
    """Dense sequences plus a paged chunk holding each one's last q_len positions."""
    H, Hkv, d, ps = 4, 2, 4, 8
    lens, q_lens = [21, 8, 5, 17], [6, 8, 1, 17]
    T = max(lens)
    q = rng.standard_normal((len(lens), H, T, d))
    rho = rng.standard_normal((len(lens), H, T, d))
    k = rng.standard_normal((len(lens), Hkv, T, d))
    v = rng.standard_normal((len(lens), Hkv, T, d))
    kp, table = _to_pages([k[b, :, :n] for b, n in enumerate(lens)], ps, rng)
    vp = np.full_like(kp, np.nan)   # V in the pages K's table names
    for b, n in enumerate(lens):
        for j in range(-(-n // ps)):
            take = min(ps, n - j * ps)
            vp[table[b, j], :, :take] = v[b, :, j * ps:j * ps + take]
    cu = np.concatenate([[0], np.cumsum(q_lens)])
    qp = np.concatenate([q[b, :, n - m:n].transpose(1, 0, 2) for b, (n, m) in enumerate(zip(lens, q_lens))])
    rp = np.concatenate([rho[b, :, n - m:n].transpose(1, 0, 2) for b, (n, m) in enumerate(zip(lens, q_lens))])
    return dict(q=q, rho=rho, k=k, v=v, qp=qp, rp=rp, kp=kp, vp=vp, table=table, cu=cu,
                lens=lens, q_lens=q_lens, H=H)


def _check_chunk_rows_equal_dense_rows(fn):
    c = _chunked_case(np.random.default_rng(11))
    rows = [(b, i, h) for b, m in enumerate(c["q_lens"]) for i in range(m) for h in range(c["H"])]
    out = fn(c["qp"], c["rp"], c["kp"], c["vp"], c["table"], c["cu"], c["lens"], rows, 0.5, causal=True)
    for (b, i, h), o in zip(rows, out):
        t = c["lens"][b] - c["q_lens"][b] + i     # a chunk's queries are the sequence's last positions
        ref = oracle.prefill_rows(c["q"][:, :, :c["lens"][b]], c["rho"][:, :, :c["lens"][b]],
                                  c["k"][:, :, :c["lens"][b]], c["v"][:, :, :c["lens"][b]],
                                  [(b, h, t)], 0.5, causal=True)[0]
        np.testing.assert_array_equal(o, ref)
    full = fn(c["qp"], c["rp"], c["kp"], c["vp"], c["table"], c["cu"], c["lens"], rows, 0.5, causal=False)
    for (b, i, h), o in zip(rows, full):
        t = c["lens"][b] - c["q_lens"][b] + i
        n = c["lens"][b]
        np.testing.assert_array_equal(
            o, oracle.parallax_query(c["q"][b, h, t], c["rho"][b, h, t], c["k"][b, h // 2, :n],
                                     c["v"][b, h // 2, :n], 0.5))


def test_paged_chunk_rows_equal_dense_prefill_rows():
    _check_chunk_rows_equal_dense_rows(oracle.prefill_paged_rows)


def test_paged_chunk_of_one_token_is_paged_decode():
    c = _chunked_case(np.random.default_rng(12))
    q1 = np.stack([c["qp"][c["cu"][b + 1] - 1] for b in range(4)])
    r1 = np.stack([c["rp"][c["cu"][b + 1] - 1] for b in range(4)])
    dec = oracle.decode(q1, r1, c["kp"], c["vp"], 0.5, seq_lens=c["lens"], page_table=c["table"])
    ones = np.arange(5)   # cu_seqlens_q of four one-token chunks
    rows = [(b, 0, h) for b in range(4) for h in range(c["H"])]
    out = oracle.prefill_paged_rows(q1.reshape(4, c["H"], -1), r1.reshape(4, c["H"], -1), c["kp"], c["vp"],
                                    c["table"], ones, c["lens"], rows, 0.5, causal=True)
    for (b, _, h), o in zip(rows, out):
        np.testing.assert_array_equal(o, dec[b, h])


def test_worked_example_as_paged_chunk():
    # The three keys of [three_keys_unequal_weights] in two 2-token pages
    # (physical order swapped); a chunk of two queries at positions 1 and 2:
    # the last sees all three keys and must give the worked answer, the
    # first sees keys 0 and 1 only.
    c = load_worked_examples()["three_keys_unequal_weights"]
    pool_k = np.full((2, 1, 2, 3), np.nan)
    pool_v = np.full((2, 1, 2, 3), np.nan)
    pool_k[1, 0, :2], pool_k[0, 0, :1] = c["k"][:2], c["k"][2:]
    pool_v[1, 0, :2], pool_v[0, 0, :1] = c["v"][:2], c["v"][2:]
    table = np.array([[1, 0]])
    q = np.stack([np.array([0.0, 0.0, 0.0]), c["q"]])[:, None]
    rho = np.stack([np.array([1.0, 0.0, 0.0]), c["rho"]])[:, None]
    out = oracle.prefill_paged_rows(q, rho, pool_k, pool_v, table, [0, 2], [3], [(0, 0, 0), (0, 1, 0)],
                                    c["scale"], causal=True)
    np.testing.assert_allclose(out[1], c["out"], atol=1e-13)
    # row 0: equal weights over keys 0, 1: vbar = (2, 4, 0), kbar = (1/2, 1/2, 0),
    # (k - kbar).rho = +1/2, -1/2; Sigma^T rho = 1/2*(1/2)(2,-4,0) + 1/2*(-1/2)(-2,4,0) = (1, -2, 0)
    np.testing.assert_allclose(out[0], [1.0, 6.0, 0.0], atol=1e-13)


def _mutant_chunk_position(q, rho, k_pool, v_pool, page_table, cu, seq_lens, rows, scale, causal=True):
    # places the chunk at the START of the sequence instead of its end
    res = []
    for b, i, h in rows:
        start = int(cu[b])
        kvh = h // (q.shape[1] // k_pool.shape[1])
        n = i + 1 if causal else int(seq_lens[b])
        K = po.gather_paged_keys(k_pool, page_table[b], n, kvh)
        V = po.gather_paged_keys(v_pool, page_table[b], n, kvh)
        res.append(po.parallax_query(q[start + i, h], rho[start + i, h], K, V, scale))
    return np.stack(res)


def _mutant_chunk_exclusive(q, rho, k_pool, v_pool, page_table, cu, seq_lens, rows, scale, causal=True):
    # the diagonal left out: query at position t sees keys 0..t-1 (and key 0 at t = 0)
    res = []
    for b, i, h in rows:
        start = int(cu[b])
        L = int(seq_lens[b])
        t = L - (int(cu[b + 1]) - start) + i
        kvh = h // (q.shape[1] // k_pool.shape[1])
        n = max(t, 1) if causal else L
        K = po.gather_paged_keys(k_pool, page_table[b], n, kvh)
        V = po.gather_paged_keys(v_pool, page_table[b], n, kvh)
        res.append(po.parallax_query(q[start + i, h], rho[start + i, h], K, V, scale))
    return np.stack(res)


@pytest.mark.parametrize("mutant", [_mutant_chunk_position, _mutant_chunk_exclusive])
def test_chunk_pin_catches_planted_mistakes(mutant):
    with pytest.raises(AssertionError):
        _check_chunk_rows_equal_dense_rows(mutant)


# --------------------------------------------------------------------------
# Mutation tests: plausible mistakes planted in the oracle must fail a pin
# --------------------------------------------------------------------------

def _mutant_transposed(q, rho, keys, values, scale):
    w = po.softmax_weights(scale * (np.asarray(keys) @ q))
    vbar = w @ values
    return vbar - po.sigma_kv(w, keys, values) @ rho        # contracts the value side


def _mutant_plus_sign(q, rho, keys, values, scale):
    w = po.softmax_weights(scale * (np.asarray(keys) @ q))
    return w @ values + po.sigma_kv(w, keys, values).T @ rho


def _mutant_uncentred(q, rho, keys, values, scale):
    w = po.softmax_weights(scale * (np.asarray(keys) @ q))
    K = np.asarray(keys)
    V = np.asarray(values)
    vbar = w @ V
    return vbar - (K.T @ (w[:, None] * V)).T @ rho          # second moment, no kbar/vbar


def _mutant_scaled_rho(q, rho, keys, values, scale):
    return po.parallax_query(q, scale * np.asarray(rho), keys, values, scale)


def _mutant_unnormalised(q, rho, keys, values, scale):
    K = np.asarray(keys)
    s = scale * (K @ q)
    w = np.exp(s - s.max())                                  # forgot the division
    vbar = w @ values
    return vbar - po.sigma_kv(w / w.sum(), keys, values).T @ rho


@pytest.mark.parametrize("mutant", [_mutant_transposed, _mutant_plus_sign, _mutant_uncentred,
                                    _mutant_scaled_rho, _mutant_unnormalised])
def test_pins_catch_planted_mistakes(mutant, monkeypatch):
    monkeypatch.setattr(oracle, "parallax_query", mutant)
    failures = 0
    for name in sorted(load_worked_examples()):
        try:
            test_worked_examples(name)
        except AssertionError:
            failures += 1
    try:
        test_solved_probe_gives_local_linear_regression(20, 4)
    except (AssertionError, ValueError):   # a shape error also exposes the mutant
        failures += 1
    assert failures > 0, f"{mutant.__name__} passed every pin"
