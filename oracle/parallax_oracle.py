"""Plain float64 definition of Parallax attention (decode and causal prefill).

TEST INFRASTRUCTURE ONLY (see the package docstring).  Every function here is
the explicit two-pass definition, written for a reader to check by eye against
the method's statement; nothing is blocked, fused or reordered.

The method ("Parallax: Breaking the Boundary Bias with Parameterized Local
Linear Attention", section "The Core Insight: Covariance Correction"): the
local linear estimate is softmax attention minus a KV-covariance term probed
by a per-query vector rho.  Written out for one query q with key set {k_i},
values {v_i}, softmax scale ``scale`` (the "bandwidth" of the newx.sg
"Abstract") and probe rho:

    w_i   = exp(s_i - max s) / sum_j exp(s_j - max s),   s_i = scale * q.k_i
    vbar  = sum_i w_i v_i                 (softmax attention, the NW estimate)
    kbar  = sum_i w_i k_i
    S_KV  = sum_i w_i (k_i - kbar)(v_i - vbar)^T          (d_k x d_v)
    out   = vbar - S_KV^T rho

Readings taken where the pages are silent or garbled (each is listed in the
design notes):
  * rho lives in key space ("query-like projector", newx.sg "Abstract"), so it
    contracts the key side of S_KV: out_j = vbar_j - sum_i w_i ((k_i-kbar).rho)
    (v_ij - vbar_j).
  * The covariance uses the same softmax weights as vbar.
  * rho is used as given: ``scale`` multiplies q.k only.
  * Causal prefill: key i is visible to query t iff i <= t.
  * Chunked prefill (a serving step the pages do not describe): the queries
    of a chunk are the last positions of their sequence, and a query at
    position t sees keys 0..t like any causal row.
  * Grouped-query attention: query head h reads KV head h // (Hq / Hkv).
  * An empty key set gives a zero output.
  * The probe is a learned linear map of the layer input ("Parallax learns it
    via a projection of the input", wispaper blog, "The Core Insight:
    Covariance Correction"): rho_h = W_R^(h) x, and likewise q_h = W_Q^(h) x,
    with no bias and no positional rotation (the pages name neither); row
    n of a weight matrix is head n // d, component n % d.  Like every
    activation of the bf16 path, q and rho are stored in bfloat16 (rounded to
    nearest, ties to even) before attention reads them.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "softmax_weights",
    "parallax_query",
    "sigma_kv",
    "decode",
    "gather_paged_keys",
    "prefill_rows",
    "prefill_paged_rows",
    "prefill_grads",
    "query_grads",
    "round_bf16",
    "project_heads",
    "decode_projected",
    "sigma_kk",
    "lla_probe",
    "lla_query",
    "lla_decode",
]


def _f64(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64)


def softmax_weights(scores) -> np.ndarray:
    """Softmax of a score vector, max-subtracted, in float64.

    Softmax attention read as a Nadaraya-Watson (local constant) estimator:
    wispaper blog, "Context: Why Softmax is Not Enough".
    """
    s = _f64(scores)
    e = np.exp(s - s.max())
    return e / e.sum()


def sigma_kv(w, keys, values) -> np.ndarray:
    """Softmax-weighted key/value cross-covariance, explicit d_k x d_v matrix.

    "KV Covariance Estimation" (newx.sg, "Innovation"); the covariance that
    the probe reads (wispaper blog, "The Core Insight").
    """
    w = _f64(w)
    K = _f64(keys)
    V = _f64(values)
    kbar = w @ K
    vbar = w @ V
    Kc = K - kbar
    Vc = V - vbar
    return Kc.T @ (w[:, None] * Vc)


def parallax_query(q, rho, keys, values, scale: float) -> np.ndarray:
    """Parallax output for one query over the key set ``keys`` [n, d_k].

    Two passes, as the definition reads: softmax weights first, then the
    explicit covariance matrix, then its product with the probe.
    (wispaper blog, "The Core Insight: Covariance Correction": output =
    softmax attention - Sigma_KV rho.)
    """
    q = _f64(q)
    rho = _f64(rho)
    K = _f64(keys)
    V = _f64(values)
    if K.shape[0] == 0:
        return np.zeros(V.shape[1], dtype=np.float64)
    w = softmax_weights(scale * (K @ q))
    vbar = w @ V
    S = sigma_kv(w, K, V)
    return vbar - S.T @ rho


def gather_paged_keys(pool, page_table_row, length: int, kv_head: int) -> np.ndarray:
    """Logical [length, d] rows of one sequence from a paged pool.

    ``pool`` is [num_pages, Hkv, page_size, d]; ``page_table_row[j]`` is the
    physical page that holds logical tokens j*page_size .. (j+1)*page_size-1.
    The oracle's own addressing; it shares nothing with the CUDA path.
    ``pool`` may be any object with ``.shape`` whose indexing returns arrays
    (so a multi-GiB pool can be read one page at a time).
    """
    page_size = pool.shape[2]
    rows = []
    n_pages = -(-length // page_size)
    for j in range(n_pages):
        page = int(page_table_row[j])
        take = min(page_size, length - j * page_size)
        rows.append(_f64(pool[page, kv_head, :take, :]))
    if not rows:
        return np.zeros((0, pool.shape[3]), dtype=np.float64)
    return np.concatenate(rows, axis=0)


def decode(q, rho, k_cache, v_cache, scale: float, seq_lens=None,
           page_table=None, heads=None):
    """Decode: one new query per (batch, query head) over its KV sequence.

    q, rho: [B, Hq, d].  Contiguous cache: k_cache, v_cache [B, Hkv, L, d],
    sequence b uses its first ``seq_lens[b]`` rows (all L when seq_lens is
    None).  Paged cache (page_table given): pools [P, Hkv, page_size, d] and
    page_table [B, max_pages].

    ``heads``: optional iterable of (b, h) to evaluate; the others are NaN.
    Returns float64 [B, Hq, d_v].
    """
    q = np.asarray(q)
    rho = np.asarray(rho)
    B, Hq, _ = q.shape
    Hkv = k_cache.shape[1]
    assert Hq % Hkv == 0
    group = Hq // Hkv
    dv = v_cache.shape[-1]
    if page_table is None:
        L = k_cache.shape[2]
    if seq_lens is None:
        assert page_table is None, "paged decode needs seq_lens"
        seq_lens = [L] * B
    out = np.full((B, Hq, dv), np.nan, dtype=np.float64)
    todo = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hq)]
    for b, h in todo:
        kvh = h // group
        n = int(seq_lens[b])
        if page_table is None:
            K = _f64(k_cache[b, kvh, :n, :])
            V = _f64(v_cache[b, kvh, :n, :])
        else:
            K = gather_paged_keys(k_cache, page_table[b], n, kvh)
            V = gather_paged_keys(v_cache, page_table[b], n, kvh)
        out[b, h] = parallax_query(q[b, h], rho[b, h], K, V, scale)
    return out


def prefill_rows(q, rho, k, v, rows, scale: float, causal: bool = True):
    """Prefill outputs for selected rows.

    q, rho: [B, H, T, d]; k, v: [B, Hkv, T, d].  Row (b, h, t) attends to keys
    0..t when ``causal`` (diagonal included), else to all T keys.
    Returns float64 [len(rows), d_v] in the order of ``rows``.  The inputs may
    be arrays or any objects with ``.shape`` whose indexing returns arrays.
    """
    H = q.shape[1]
    Hkv = k.shape[1]
    group = H // Hkv
    T = k.shape[2]
    res = []
    for b, h, t in rows:
        kvh = h // group
        n = t + 1 if causal else T
        res.append(parallax_query(q[b, h, t], rho[b, h, t],
                                  k[b, kvh, :n, :], v[b, kvh, :n, :], scale))
    return np.stack(res) if res else np.zeros((0, v.shape[-1]))


def prefill_paged_rows(q, rho, k_pool, v_pool, page_table, cu_seqlens_q, seq_lens, rows,
                       scale: float, causal: bool = True):
    """Chunked (append) prefill over a paged cache, for selected rows.

    Sequence b holds ``seq_lens[b]`` keys in the pools [P, Hkv, page_size, d]
    through ``page_table[b]``.  Its q_len = cu_seqlens_q[b+1] - cu_seqlens_q[b]
    queries are packed in q, rho [total_q, H, d] from row cu_seqlens_q[b] and
    are the sequence's last positions: query i sits at position
    t = seq_lens[b] - q_len + i and attends to keys 0..t when ``causal``,
    else to all seq_lens[b] keys.  ``rows``: iterable of (b, i, h).
    Returns float64 [len(rows), d_v] in the order of ``rows``.
    """
    H = q.shape[1]
    Hkv = k_pool.shape[1]
    group = H // Hkv
    gathered = {}
    res = []
    for b, i, h in rows:
        start = int(cu_seqlens_q[b])
        q_len = int(cu_seqlens_q[b + 1]) - start
        L = int(seq_lens[b])
        assert 0 <= i < q_len <= L, (b, i, q_len, L)
        t = L - q_len + i
        n = t + 1 if causal else L
        kvh = h // group
        if (b, kvh) not in gathered:
            gathered[(b, kvh)] = (gather_paged_keys(k_pool, page_table[b], L, kvh),
                                  gather_paged_keys(v_pool, page_table[b], L, kvh))
        K, V = gathered[(b, kvh)]
        res.append(parallax_query(q[start + i, h], rho[start + i, h], K[:n], V[:n], scale))
    return np.stack(res) if res else np.zeros((0, v_pool.shape[-1]))


def _prefill_out_torch(Q, R, K, V, scale: float, causal: bool):
    """out of one (sequence, head) prefill from torch float64 tensors [T, d]:
    softmax weights, the explicit d x d covariance of every row, its product
    with the probe (the definition of ``parallax_query``, one row per t)."""
    import torch
    T = Q.shape[0]
    s = scale * Q @ K.T
    if causal:
        s = s.masked_fill(torch.triu(torch.ones(T, T, dtype=torch.bool), diagonal=1), float("-inf"))
    w = torch.softmax(s, dim=-1)                                   # [T, T]
    vbar = w @ V
    kbar = w @ K
    kc = K[None, :, :] - kbar[:, None, :]                          # [T, T, d]
    vc = V[None, :, :] - vbar[:, None, :]
    sigma = torch.einsum("ti,tid,tie->tde", w, kc, vc)             # d_k x d_v per row
    return vbar - torch.einsum("tde,td->te", sigma, R)


def prefill_grads(q, rho, k, v, dout, scale: float, causal: bool = True):
    """Gradients of sum(dout * out) for a prefill, in float64.

    q, rho, dout: [B, H, T, d]; k, v: [B, Hkv, T, d].  ``out`` is built by
    ``_prefill_out_torch`` from torch float64 tensors, and torch's
    reverse-mode autograd (a library routine) differentiates it.  Returns
    (dq, drho, dk, dv) as float64 numpy arrays shaped like the inputs.
    """
    import torch

    def t(x):
        return torch.tensor(np.asarray(x, dtype=np.float64), dtype=torch.float64, requires_grad=True)

    Q, R, K, V = t(q), t(rho), t(k), t(v)
    G = torch.tensor(np.asarray(dout, dtype=np.float64), dtype=torch.float64)
    B, H = Q.shape[:2]
    group = H // K.shape[1]
    total = torch.zeros((), dtype=torch.float64)
    for b in range(B):
        for h in range(H):
            out = _prefill_out_torch(Q[b, h], R[b, h], K[b, h // group], V[b, h // group], scale, causal)
            total = total + (out * G[b, h]).sum()
    total.backward()
    return tuple(x.grad.numpy() for x in (Q, R, K, V))


def query_grads(q, rho, keys, values, dout, scale: float):
    """Gradients of dout . out for ONE query over the key set ``keys`` [n, d]
    (the row of ``parallax_query``): returns (dq, drho, dkeys, dvalues) as
    float64 numpy arrays.  Same construction as ``prefill_grads`` (torch
    float64 autograd through the explicit covariance), for one row, so a
    long prefill can be checked on sampled rows and keys."""
    import torch

    def t(x):
        return torch.tensor(np.asarray(x, dtype=np.float64), dtype=torch.float64, requires_grad=True)

    Q, R, K, V = t(np.asarray(q)[None]), t(np.asarray(rho)[None]), t(keys), t(values)
    G = torch.tensor(np.asarray(dout, dtype=np.float64)[None], dtype=torch.float64)
    w = torch.softmax(scale * Q @ K.T, dim=-1)                        # [1, n]
    vbar = w @ V
    kbar = w @ K
    sigma = torch.einsum("ti,tid,tie->tde", w, K[None] - kbar[:, None], V[None] - vbar[:, None])
    out = vbar - torch.einsum("tde,td->te", sigma, R)
    (out * G).sum().backward()
    return Q.grad.numpy()[0], R.grad.numpy()[0], K.grad.numpy(), V.grad.numpy()


# --------------------------------------------------------------- projection

_BF16_MIN_ULP = 2.0 ** -133          # spacing of the subnormal bfloat16 values
_BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127


def round_bf16(x) -> np.ndarray:
    """float64 values rounded to the nearest bfloat16, ties to even, returned
    as float64.

    bfloat16 is float32 with 8 significant bits: a value with leading bit
    2^(e-1) (``numpy.frexp`` gives x = m 2^e, 1/2 <= |m| < 1) has spacing
    2^(e-8), never below the subnormal spacing 2^-133.  x / spacing is exact
    in float64; ``numpy.round`` takes it to the nearest integer with ties to
    even; magnitudes past the largest finite bfloat16 become infinite.
    NaN stays NaN.
    """
    x = _f64(x)
    _, e = np.frexp(x)
    ulp = np.maximum(np.ldexp(1.0, e - 8), _BF16_MIN_ULP)
    with np.errstate(invalid="ignore"):
        y = np.round(x / ulp) * ulp
        y = np.where(np.abs(y) > _BF16_MAX, np.copysign(np.inf, x), y)
    return np.where(np.isfinite(x), y, x)


def project_heads(x, weight, num_heads: int, head_dim: int) -> np.ndarray:
    """Per-head linear projection of the layer input, in float64:
    y[b, h, j] = sum_c weight[h * head_dim + j, c] * x[b, c].

    x: [B, hidden]; weight: [num_heads * head_dim, hidden] (output feature
    by input feature).  Returns float64 [B, num_heads, head_dim], unrounded.
    """
    x = _f64(x)
    weight = _f64(weight)
    assert weight.shape == (num_heads * head_dim, x.shape[1])
    return (x @ weight.T).reshape(x.shape[0], num_heads, head_dim)


def decode_projected(x, w_q, w_rho, k_cache, v_cache, scale: float, seq_lens=None,
                     page_table=None, heads=None):
    """Decode whose query and probe come from the new token's layer input:
    q = bf16(W_Q x), rho = bf16(W_R x) per head (``project_heads`` then
    ``round_bf16``), then ``decode``.

    x: [B, hidden]; w_q, w_rho: [Hq * d, hidden]; caches as in ``decode``.
    Returns (q, rho, out): the rounded projections [B, Hq, d] and the float64
    output [B, Hq, d_v].
    """
    d = k_cache.shape[-1]
    Hq = np.asarray(w_q).shape[0] // d
    q = round_bf16(project_heads(x, w_q, Hq, d))
    rho = round_bf16(project_heads(x, w_rho, Hq, d))
    return q, rho, decode(q, rho, k_cache, v_cache, scale, seq_lens=seq_lens,
                          page_table=page_table, heads=heads)


# ------------------------------------------------- LLA with the solved probe

def sigma_kk(w, keys) -> np.ndarray:
    """Softmax-weighted key covariance, explicit d_k x d_k matrix:
    sum_i w_i (k_i - kbar)(k_i - kbar)^T with kbar = sum_i w_i k_i."""
    w = _f64(w)
    K = _f64(keys)
    Kc = K - w @ K
    return Kc.T @ (w[:, None] * Kc)


def lla_probe(q, keys, scale: float, ridge: float) -> np.ndarray:
    """The probe Local Linear Attention solves for, per query.

    LLA is the local linear estimate: the intercept of the softmax-weighted
    least-squares fit v ~ a + M^T (k - q) (newx.sg "Abstract": it upgrades
    the local constant estimate of softmax attention to a local linear one;
    wispaper blog, "Context: Why Softmax is Not Enough": it solves a linear
    system for every token).  Its intercept is vbar - S_KV^T rho* with
        (S_KK + ridge I) rho* = kbar - q,
    where ``ridge`` >= 0 penalises the slope M (ridge * ||M||^2; the pages
    name no regularisation, so it is a parameter and 0 is plain LLA).  The
    system is solved exactly (numpy.linalg.solve); the pages' solver is
    conjugate gradients, whose converged answer is the same.  An empty key
    set gives rho* = 0.
    """
    q = _f64(q)
    K = _f64(keys)
    if K.shape[0] == 0:
        return np.zeros(K.shape[1], dtype=np.float64)
    w = softmax_weights(scale * (K @ q))
    kbar = w @ K
    A = sigma_kk(w, K) + ridge * np.eye(K.shape[1])
    return np.linalg.solve(A, kbar - q)


def lla_query(q, keys, values, scale: float, ridge: float):
    """LLA output for one query: (rho*, vbar - S_KV^T rho*), the Parallax
    output of ``parallax_query`` with the solved probe in place of a learned
    one."""
    rho = lla_probe(q, keys, scale, ridge)
    return rho, parallax_query(q, rho, keys, values, scale)


def lla_decode(q, k_cache, v_cache, scale: float, ridge: float, seq_lens=None, page_table=None, heads=None):
    """Decode with LLA's solved probe: for every (sequence, query head),
    ``lla_query`` over the sequence's keys (contiguous or paged caches, GQA
    and ``heads`` as in ``decode``).  Returns (rho*, out), float64
    [B, Hq, d_k] and [B, Hq, d_v]; heads not evaluated are NaN."""
    q = np.asarray(q)
    B, Hq, dk = q.shape
    Hkv = k_cache.shape[1]
    group = Hq // Hkv
    dv = v_cache.shape[-1]
    if seq_lens is None:
        assert page_table is None, "paged decode needs seq_lens"
        seq_lens = [k_cache.shape[2]] * B
    rho = np.full((B, Hq, dk), np.nan, dtype=np.float64)
    out = np.full((B, Hq, dv), np.nan, dtype=np.float64)
    todo = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hq)]
    for b, h in todo:
        kvh = h // group
        n = int(seq_lens[b])
        if page_table is None:
            K = _f64(k_cache[b, kvh, :n, :])
            V = _f64(v_cache[b, kvh, :n, :])
        else:
            K = gather_paged_keys(k_cache, page_table[b], n, kvh)
            V = gather_paged_keys(v_cache, page_table[b], n, kvh)
        rho[b, h], out[b, h] = lla_query(q[b, h], K, V, scale, ridge)
    return rho, out

