"""Pins of the oracle's projected decode (q and rho projected from the layer
input, then rounded to bfloat16) to facts fixed outside the oracle.

``round_bf16`` is checked against torch's float32 -> bfloat16 cast (the same
rounding where the input is a float32) and against hand-picked ties;
``project_heads`` against permutation and single-entry weights, whose
results are known without a matrix product; ``decode_projected`` against
softmax attention when the probe weights vanish.  The mutation test at the end
plants plausible mistakes into the oracle and checks that the pins catch them.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import parallax_oracle as po

RNG = np.random.default_rng(20261202)


# --------------------------------------------------------------------------
# bfloat16 rounding
# --------------------------------------------------------------------------

def test_round_bf16_equals_torch_cast_on_float32_values():
    # float32 values over the whole exponent range, subnormals included:
    # there torch's cast is the same round-to-nearest-even.
    mant = RNG.standard_normal(200_000).astype(np.float32)
    expo = RNG.integers(-149, 128, 200_000)
    with np.errstate(over="ignore"):
        x = np.ldexp(mant.astype(np.float64), expo).astype(np.float32)
    x = x[np.isfinite(x)]
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.round_bf16(x.astype(np.float64)), want)


@pytest.mark.parametrize("x, want", [
    (1.0 + 2.0 ** -8, 1.0),                        # tie, even neighbour below
    (1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -6),        # tie, even neighbour above
    (-(1.0 + 2.0 ** -8), -1.0),
    (1.0 + 2.0 ** -8 + 2.0 ** -40, 1.0 + 2.0 ** -7),   # just past the tie (not a float32)
    (255.5, 256.0),                                # tie at 8 significant bits
    (1.5 * 2.0 ** -133, 2.0 ** -132),              # subnormal tie, to even
    (0.5 * 2.0 ** -133, 0.0),                      # half the smallest subnormal, to even
    ((2.0 - 2.0 ** -8) * 2.0 ** 127, np.inf),      # halfway past the largest finite
    ((2.0 - 2.0 ** -7) * 2.0 ** 127, (2.0 - 2.0 ** -7) * 2.0 ** 127),
])
def test_round_bf16_ties_and_limits(x, want):
    assert oracle.round_bf16(np.array([x]))[0] == want


# --------------------------------------------------------------------------
# Per-head projection
# --------------------------------------------------------------------------

def test_project_heads_permutation_weight():
    # W = permutation matrix: y[b, n] = x[b, perm[n]] exactly, with n = h*d + j.
    # A transposed weight would read x[b, perm^-1[n]] instead.
    H, d, B = 3, 8, 4
    n = H * d
    perm = RNG.permutation(n)
    assert not np.array_equal(perm[perm], np.arange(n))     # not an involution
    W = np.zeros((n, n))
    W[np.arange(n), perm] = 1.0
    x = RNG.standard_normal((B, n))
    y = oracle.project_heads(x, W, H, d)
    for b in range(B):
        for h in range(H):
            for j in range(d):
                assert y[b, h, j] == x[b, perm[h * d + j]]


def test_project_heads_single_entry_places_head_and_component():
    H, d, hidden = 4, 8, 12
    h0, j0, c0 = 2, 5, 7
    W = np.zeros((H * d, hidden))
    W[h0 * d + j0, c0] = 3.0
    x = RNG.standard_normal((2, hidden))
    y = oracle.project_heads(x, W, H, d)
    want = np.zeros_like(y)
    want[:, h0, j0] = 3.0 * x[:, c0]
    np.testing.assert_array_equal(y, want)


def test_projection_rounds_the_exact_sum_once():
    # x . w = 1 + 2^-8 exactly: a bfloat16 tie, which goes to 1.0.  In the
    # second row the sum passes through 3 + 2^-8 + 2^-30 before the -2:
    # rounding that partial sum to bfloat16 would give 3, and then 1.0,
    # instead of the 1 + 2^-7 that the exact sum rounds to.
    d, hidden = 2, 3
    x = np.array([[1.0, 2.0 ** -8, 0.0], [3.0, 2.0 ** -8 + 2.0 ** -30, -2.0]])
    W = np.array([[1.0, 1.0, 0.0], [1.0, 1.0, 1.0]])
    y = oracle.round_bf16(oracle.project_heads(x, W, 1, d))
    assert y[0, 0, 0] == 1.0 and y[0, 0, 1] == 1.0
    # 3 + 2^-8 + 2^-30 - 2 = 1 + 2^-8 + 2^-30: just past the tie, rounds up
    assert y[1, 0, 1] == 1.0 + 2.0 ** -7


# --------------------------------------------------------------------------
# Projected decode
# --------------------------------------------------------------------------

def test_decode_projected_with_zero_probe_weights_is_softmax_attention():
    B, Hq, Hkv, d, L, hidden = 2, 4, 2, 16, 9, 24
    x = RNG.standard_normal((B, hidden))
    w_q = RNG.standard_normal((Hq * d, hidden)) / np.sqrt(hidden)
    w_rho = np.zeros_like(w_q)
    k = RNG.standard_normal((B, Hkv, L, d))
    v = RNG.standard_normal((B, Hkv, L, d))
    scale = 0.25
    q, rho, out = oracle.decode_projected(x, w_q, w_rho, k, v, scale)
    assert not rho.any()
    g = Hq // Hkv
    kk = torch.from_numpy(np.repeat(k, g, axis=1))
    vv = torch.from_numpy(np.repeat(v, g, axis=1))
    want = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[:, :, None], kk, vv, scale=scale)[:, :, 0].numpy()
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-12)


def test_decode_projected_permutation_weights_pass_x_through():
    # hidden = Hq * d and permutation weights: q and rho are permuted copies of
    # the (bfloat16-exact) input, so the output is decode() on those copies.
    B, Hq, Hkv, d, L = 2, 2, 1, 8, 5
    n = Hq * d
    x = oracle.round_bf16(RNG.standard_normal((B, n)))
    pq, pr = RNG.permutation(n), RNG.permutation(n)
    w_q = np.zeros((n, n))
    w_q[np.arange(n), pq] = 1.0
    w_rho = np.zeros((n, n))
    w_rho[np.arange(n), pr] = 1.0
    k = RNG.standard_normal((B, Hkv, L, d))
    v = RNG.standard_normal((B, Hkv, L, d))
    q, rho, out = oracle.decode_projected(x, w_q, w_rho, k, v, 0.3)
    np.testing.assert_array_equal(q.reshape(B, n), x[:, pq])
    np.testing.assert_array_equal(rho.reshape(B, n), x[:, pr])
    np.testing.assert_array_equal(out, oracle.decode(q, rho, k, v, 0.3))


# --------------------------------------------------------------------------
# Planted mistakes
# --------------------------------------------------------------------------

def _proj_transposed(x, weight, num_heads, head_dim):
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(weight, dtype=np.float64)
    return (x @ w).reshape(x.shape[0], num_heads, head_dim)


def _proj_head_major_swap(x, weight, num_heads, head_dim):
    # component-major instead of head-major output features
    y = np.asarray(x, dtype=np.float64) @ np.asarray(weight, dtype=np.float64).T
    return y.reshape(y.shape[0], head_dim, num_heads).transpose(0, 2, 1)


def _round_half_up(x):
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    ulp = np.maximum(np.ldexp(1.0, e - 8), 2.0 ** -133)
    return np.floor(x / ulp + 0.5) * ulp


def _round_truncate(x):
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    ulp = np.maximum(np.ldexp(1.0, e - 8), 2.0 ** -133)
    return np.trunc(x / ulp) * ulp


PINS = [
    test_project_heads_permutation_weight,
    test_project_heads_single_entry_places_head_and_component,
    test_projection_rounds_the_exact_sum_once,
    test_decode_projected_permutation_weights_pass_x_through,
    test_round_bf16_equals_torch_cast_on_float32_values,
]


@pytest.mark.parametrize("name, mutant", [
    ("project_heads", _proj_transposed),
    ("project_heads", _proj_head_major_swap),
    ("round_bf16", _round_half_up),
    ("round_bf16", _round_truncate),
])
def test_projection_pins_catch_planted_mistakes(name, mutant, monkeypatch):
    monkeypatch.setattr(po, name, mutant)
    monkeypatch.setattr(oracle, name, mutant)
    caught = 0
    for pin in PINS:
        try:
            pin()
        except (AssertionError, ValueError):
            caught += 1
    if name == "round_bf16":
        with pytest.raises(AssertionError):
            for x, want in [(1.0 + 2.0 ** -8, 1.0), (1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -6),
                            (-(1.0 + 2.0 ** -8), -1.0)]:
                assert oracle.round_bf16(np.array([x]))[0] == want
    else:
        assert caught > 0


def test_decode_projected_paged_equals_contiguous():
    # the same logical cache stored in pages placed by a permutation
    from parallax_local_linear_b200 import workloads as W
    inp = W.small_decode_inputs(3, 4, 2, 64, 150, seq_lens=[150, 1, 77], paged=True, seed=12,
                                nan_poison=True)
    pj = W.projection_inputs(3, 4, 64, 96, seed=13)
    args = [pj[k].double().numpy() for k in ("x", "w_q", "w_rho")]
    lens = inp["seq_lens"].numpy()
    _, _, paged = oracle.decode_projected(*args, inp["k_cache"].double().numpy(), inp["v_cache"].double().numpy(),
                                          inp["scale"], seq_lens=lens, page_table=inp["page_table"].numpy())
    _, _, contig = oracle.decode_projected(*args, inp["k_contig"].double().numpy(),
                                           inp["v_contig"].double().numpy(), inp["scale"], seq_lens=lens)
    np.testing.assert_array_equal(paged, contig)
