"""Seeded synthetic inputs for Parallax decode and prefill.

This module only draws and lays out inputs; it holds none of the method's
arithmetic, and both the CUDA path and the float64 oracle consume what it
returns.  Values are drawn as float32 with a torch generator seeded per
workload (on the device that will hold them, so multi-GiB caches never cross
PCIe), then rounded to bfloat16 with round-to-nearest-even.  The oracle reads
back the very same rounded values.

Named workloads (head_dim d, Hq query heads, Hkv KV heads):
  decode_f32     B=1,   Hq=1,  Hkv=1, d=64,  L=256,   float32 throughout
  decode_bf16    B=8,   Hq=16, Hkv=8, d=128, L=4096,  contiguous cache
  decode_long    B=64,  Hq=32, Hkv=8, d=128, L=32768, keys offset per KV head
  decode_paged   128 sequences, L ~ U{512..65536}, Hq=16, Hkv=4, d=128,
                 64-token pages placed by a seeded permutation
  lla_decode     decode_bf16's inputs through Local Linear Attention with the
                 solved probe (ridge 0)
  prefill        B=4, H=16, T=8192, d=128, causal, rho scaled by 0.1
  prefill_train  the same shapes, forward for training plus backward, with
                 dL/dout ~ N(0, 1)
  prefill_paged  chunked (append) prefill over a paged cache: 8 sequences,
                 H=16, Hkv=4, d=128; each appends a chunk of U{1024..4096}
                 queries to a cached prefix of U{0..8192} tokens; 64-token
                 pages placed by a seeded permutation; rho scaled by 0.1
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

PAGE_SIZE = 64


@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    kv_len: int
    dtype: str = "bf16"           # "bf16" or "f32"
    key_offset_std: float = 0.0   # per-KV-head offset added to every key
    paged: bool = False
    min_len: int = 0              # paged: lengths uniform in [min_len, kv_len]
    seed: int = 0
    hidden: int = 0               # > 0: q and rho are projected from a [B, hidden] input

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


@dataclass(frozen=True)
class PrefillWorkload:
    name: str
    batch: int
    num_heads: int
    seq_len: int
    head_dim: int
    num_kv_heads: int = 0
    rho_scale: float = 0.1
    causal: bool = True
    seed: int = 0

    @property
    def kv_heads(self) -> int:
        return self.num_kv_heads or self.num_heads

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


@dataclass(frozen=True)
class ChunkedPrefillWorkload:
    name: str
    batch: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    q_min: int          # chunk lengths uniform in [q_min, q_max]
    q_max: int
    prefix_max: int     # cached prefix lengths uniform in [0, prefix_max]
    rho_scale: float = 0.1
    causal: bool = True
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)


WORKLOADS = {
    "decode_f32": DecodeWorkload("decode_f32", 1, 1, 1, 64, 256, dtype="f32", seed=1),
    "decode_bf16": DecodeWorkload("decode_bf16", 8, 16, 8, 128, 4096, seed=2),
    # decode_bf16's cache with q and rho projected from a model width of Hq * d
    "decode_projected": DecodeWorkload("decode_projected", 8, 16, 8, 128, 4096, seed=2, hidden=2048),
    "decode_long": DecodeWorkload("decode_long", 64, 32, 8, 128, 32768, key_offset_std=0.5, seed=3),
    "decode_paged": DecodeWorkload("decode_paged", 128, 16, 4, 128, 65536, paged=True,
                                   min_len=512, seed=4),
    # decode_bf16's cache and queries through Local Linear Attention with the solved probe
    "lla_decode": DecodeWorkload("lla_decode", 8, 16, 8, 128, 4096, seed=2),
    "prefill": PrefillWorkload("prefill", 4, 16, 8192, 128, seed=5),
    "prefill_train": PrefillWorkload("prefill_train", 4, 16, 8192, 128, seed=5),
    "prefill_paged": ChunkedPrefillWorkload("prefill_paged", 8, 16, 4, 128, 1024, 4096, 8192, seed=6),
}


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal(shape, gen, device, out_dtype, chunk_dim0=True, add=None, mul=1.0):
    """float32 N(0,1) draws, optionally scaled / offset, rounded to out_dtype.

    Large tensors are drawn one leading-index slice at a time so the float32
    staging copy stays small.
    """
    out = torch.empty(shape, dtype=out_dtype, device=device)
    if chunk_dim0 and len(shape) > 1 and out.numel() > (1 << 26):
        for i in range(shape[0]):
            x = torch.randn(shape[1:], generator=gen, device=device, dtype=torch.float32)
            if mul != 1.0:
                x.mul_(mul)
            if add is not None:
                x.add_(add)
            out[i].copy_(x)
        return out
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if mul != 1.0:
        x.mul_(mul)
    if add is not None:
        x.add_(add)
    out.copy_(x)
    return out


def paged_layout(batch, kv_len, min_len, seed, page_size=PAGE_SIZE):
    """Sequence lengths, page count and page table of a ragged paged cache.

    Lengths are integers uniform in [min_len, kv_len] (both ends included);
    the pool has sum(ceil(L_b / page_size)) pages; a seeded permutation of the
    pool gives each sequence its pages in order.  Unused table slots are -1.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    lens = rng.integers(min_len, kv_len + 1, size=batch).astype(np.int32)
    n_pages = -(-lens.astype(np.int64) // page_size)
    total = int(n_pages.sum())
    perm = rng.permutation(total).astype(np.int32)
    max_pages = int(-(-kv_len // page_size))
    table = np.full((batch, max_pages), -1, dtype=np.int32)
    cur = 0
    for b in range(batch):
        table[b, : n_pages[b]] = perm[cur: cur + n_pages[b]]
        cur += int(n_pages[b])
    return lens, table, total


def decode_inputs(w: DecodeWorkload, device="cpu", seed=None, nan_poison=True):
    """Inputs of one decode call.

    Returns a dict: q, rho [B, Hq, d]; k_cache, v_cache ([B, Hkv, L, d] or
    the paged pool [P, Hkv, 64, d]); seq_lens (int32 [B] or None);
    page_table (int32 [B, max_pages] or None); scale.  With ``nan_poison``
    the unused tail of every last page is NaN, so any over-read shows.
    """
    seed = w.seed if seed is None else seed
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    gen = _gen(device, seed)
    B, Hq, Hkv, d = w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim
    q = _normal((B, Hq, d), gen, device, dt)
    rho = _normal((B, Hq, d), gen, device, dt)
    seq_lens = page_table = None
    if w.paged:
        lens, table, total = paged_layout(B, w.kv_len, w.min_len, seed)
        shape = (total, Hkv, PAGE_SIZE, d)
    else:
        shape = (B, Hkv, w.kv_len, d)
    offset = None
    if w.key_offset_std:
        # one d-vector per KV head, shared by every sequence and position
        offset = (torch.randn((Hkv, d), generator=gen, device=device, dtype=torch.float32)
                  * w.key_offset_std)
    k = torch.empty(shape, dtype=dt, device=device)
    v = torch.empty(shape, dtype=dt, device=device)
    for i in range(shape[0]):
        x = torch.randn(shape[1:], generator=gen, device=device, dtype=torch.float32)
        if offset is not None:
            x.add_(offset[:, None, :])
        k[i].copy_(x)
    for i in range(shape[0]):
        v[i].copy_(torch.randn(shape[1:], generator=gen, device=device, dtype=torch.float32))
    if w.paged:
        seq_lens = torch.from_numpy(lens).to(device)
        page_table = torch.from_numpy(table).to(device)
        if nan_poison:
            _poison_paged_tails(k, v, lens, table)
    return dict(q=q, rho=rho, k_cache=k, v_cache=v, seq_lens=seq_lens,
                page_table=page_table, scale=w.scale)


def projection_inputs(batch, num_q_heads, head_dim, hidden, device="cpu", seed=0):
    """Layer input and projection weights of a projected decode.

    x [B, hidden] ~ N(0, 1); w_q, w_rho [Hq * d, hidden] ~ N(0, 1 / hidden)
    (so every projected component has unit variance, like the q and rho
    draws of the plain decode inputs); all rounded to bfloat16.  Drawn from
    their own generator, seeded ``seed``, in the order x, w_q, w_rho.
    """
    gen = _gen(device, seed)
    n = num_q_heads * head_dim
    x = _normal((batch, hidden), gen, device, torch.bfloat16)
    w_q = _normal((n, hidden), gen, device, torch.bfloat16, mul=hidden ** -0.5)
    w_rho = _normal((n, hidden), gen, device, torch.bfloat16, mul=hidden ** -0.5)
    return dict(x=x, w_q=w_q, w_rho=w_rho)


def projected_decode_inputs(w: DecodeWorkload, device="cpu", seed=None):
    """Inputs of one projected decode call: ``decode_inputs`` (its q and rho
    unused) plus ``projection_inputs`` drawn with seed + 104729."""
    seed = w.seed if seed is None else seed
    inp = decode_inputs(w, device=device, seed=seed)
    inp.update(projection_inputs(w.batch, w.num_q_heads, w.head_dim, w.hidden, device=device,
                                 seed=seed + 104729))
    return inp


def projection_bytes(batch, num_q_heads, head_dim, hidden) -> int:
    """Bytes a projected decode moves beyond the KV cache: both weight
    matrices and x read once, q and rho written once (bf16)."""
    n = num_q_heads * head_dim
    return 2 * (2 * n * hidden + batch * hidden + 2 * batch * n)


def _poison_paged_tails(k, v, lens, table, page_size=PAGE_SIZE):
    for b, n in enumerate(lens):
        n = int(n)
        if n % page_size:
            last = int(table[b, (n - 1) // page_size])
            k[last, :, n % page_size:, :] = float("nan")
            v[last, :, n % page_size:, :] = float("nan")


def small_decode_inputs(batch, num_q_heads, num_kv_heads, head_dim, kv_len, *, dtype="bf16",
                        seq_lens=None, paged=False, page_size=PAGE_SIZE, key_offset_std=0.0,
                        seed=0, device="cpu", nan_poison=True, value_offset=0.0):
    """Decode inputs of arbitrary (small) shape for parity sweeps.

    ``seq_lens``: optional list of lengths (each <= kv_len).  Contiguous
    caches have their rows past each length set to NaN (with nan_poison).
    ``paged``: the same logical cache, stored in pages placed by a seeded
    permutation; returns the contiguous copy too (keys ``k_contig``,
    ``v_contig``) so the two layouts can be compared.
    """
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    gen = _gen("cpu", seed)
    B, Hq, Hkv, d, L = batch, num_q_heads, num_kv_heads, head_dim, kv_len
    q = torch.randn((B, Hq, d), generator=gen).to(dt)
    rho = torch.randn((B, Hq, d), generator=gen).to(dt)
    kx = torch.randn((B, Hkv, L, d), generator=gen)
    if key_offset_std:
        kx += torch.randn((Hkv, d), generator=gen)[None, :, None, :] * key_offset_std
    vx = torch.randn((B, Hkv, L, d), generator=gen) + value_offset
    k = kx.to(dt)
    v = vx.to(dt)
    lens = None if seq_lens is None else torch.tensor(seq_lens, dtype=torch.int32)
    if lens is not None and nan_poison:
        for b, n in enumerate(seq_lens):
            k[b, :, n:] = float("nan")
            v[b, :, n:] = float("nan")
    res = dict(q=q, rho=rho, k_cache=k, v_cache=v, seq_lens=lens, page_table=None,
               scale=1.0 / math.sqrt(d))
    if paged:
        lens_list = list(seq_lens) if seq_lens is not None else [L] * B
        n_pages = [-(-n // page_size) for n in lens_list]
        total = max(1, sum(n_pages))
        rng = np.random.Generator(np.random.PCG64(seed + 7))
        perm = rng.permutation(total)
        max_pages = max(1, -(-L // page_size))
        table = np.full((B, max_pages), -1, dtype=np.int32)
        kp = torch.full((total, Hkv, page_size, d), float("nan"), dtype=dt)
        vp = torch.full((total, Hkv, page_size, d), float("nan"), dtype=dt)
        cur = 0
        for b, n in enumerate(lens_list):
            for j in range(n_pages[b]):
                page = int(perm[cur])
                cur += 1
                table[b, j] = page
                take = min(page_size, n - j * page_size)
                kp[page, :, :take] = k[b, :, j * page_size: j * page_size + take]
                vp[page, :, :take] = v[b, :, j * page_size: j * page_size + take]
        res.update(k_contig=k, v_contig=v, k_cache=kp, v_cache=vp,
                   page_table=torch.from_numpy(table),
                   seq_lens=torch.tensor(lens_list, dtype=torch.int32))
    return res


def prefill_inputs(w: PrefillWorkload, device="cpu", seed=None):
    """q, rho [B, H, T, d]; k, v [B, Hkv, T, d] (bfloat16); rho scaled by rho_scale."""
    seed = w.seed if seed is None else seed
    gen = _gen(device, seed)
    B, H, T, d = w.batch, w.num_heads, w.seq_len, w.head_dim
    q = _normal((B, H, T, d), gen, device, torch.bfloat16)
    rho = _normal((B, H, T, d), gen, device, torch.bfloat16, mul=w.rho_scale)
    k = _normal((B, w.kv_heads, T, d), gen, device, torch.bfloat16)
    v = _normal((B, w.kv_heads, T, d), gen, device, torch.bfloat16)
    return dict(q=q, rho=rho, k=k, v=v, scale=w.scale, causal=w.causal)


def small_prefill_inputs(batch, num_heads, seq_len, head_dim, *, num_kv_heads=0, rho_scale=0.1,
                         seed=0, device="cpu"):
    w = PrefillWorkload("small", batch, num_heads, seq_len, head_dim,
                        num_kv_heads=num_kv_heads, rho_scale=rho_scale, seed=seed)
    return prefill_inputs(w, device=device)


def kv_bytes(w: DecodeWorkload, seq_lens=None) -> int:
    """Algorithmic K+V bytes one decode call reads: every row once."""
    elt = 4 if w.dtype == "f32" else 2
    if seq_lens is None:
        tokens = w.batch * w.kv_len
    else:
        tokens = int(np.asarray(seq_lens, dtype=np.int64).sum())
    return tokens * w.num_kv_heads * 2 * w.head_dim * elt


def prefill_flops(w: PrefillWorkload) -> int:
    """Algorithmic FLOP of one prefill call: 8*d per visible (query, key) pair
    (q.k, rho.k, and the two weighted value products, 2*d each)."""
    T = w.seq_len
    pairs = T * (T + 1) // 2 if w.causal else T * T
    return 8 * w.head_dim * pairs * w.batch * w.num_heads



def chunked_layout(q_lens, prefix_lens, seed, page_size=PAGE_SIZE):
    """Offsets, lengths and page table of chunks appended to cached prefixes.

    Sequence b holds prefix_lens[b] + q_lens[b] keys; its chunk is packed at
    rows cu[b] .. cu[b+1]-1.  Pages come from a seeded permutation of a pool
    of sum(ceil(L_b / page_size)) pages (at least one); unused slots are -1.
    """
    q_lens = np.asarray(q_lens, dtype=np.int64)
    lens = q_lens + np.asarray(prefix_lens, dtype=np.int64)
    cu = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    n_pages = -(-lens // page_size)
    total = max(1, int(n_pages.sum()))
    perm = np.random.Generator(np.random.PCG64(seed)).permutation(total).astype(np.int32)
    table = np.full((len(lens), max(1, int(n_pages.max(initial=0)))), -1, dtype=np.int32)
    cur = 0
    for b, n in enumerate(n_pages):
        table[b, :n] = perm[cur: cur + n]
        cur += int(n)
    return cu, lens.astype(np.int32), table, total


def chunked_prefill_inputs(w: ChunkedPrefillWorkload, device="cpu", seed=None, nan_poison=True):
    """Inputs of one chunked prefill call.

    Returns a dict: q, rho [total_q, H, d] bf16 (rho scaled by rho_scale);
    pools k_cache, v_cache [P, Hkv, 64, d] bf16; page_table, cu_seqlens_q,
    seq_lens (int32, on ``device``); their host copies q_lens, seq_lens_host;
    max_q_len; scale; causal.  With ``nan_poison`` the unused tail of every
    last page is NaN.
    """
    seed = w.seed if seed is None else seed
    rng = np.random.Generator(np.random.PCG64(seed))
    q_lens = rng.integers(w.q_min, w.q_max + 1, size=w.batch)
    prefix = rng.integers(0, w.prefix_max + 1, size=w.batch)
    cu, lens, table, total = chunked_layout(q_lens, prefix, seed + 1)
    gen = _gen(device, seed)
    H, Hkv, d = w.num_heads, w.num_kv_heads, w.head_dim
    tq = int(cu[-1])
    q = _normal((tq, H, d), gen, device, torch.bfloat16)
    rho = _normal((tq, H, d), gen, device, torch.bfloat16, mul=w.rho_scale)
    k = _normal((total, Hkv, PAGE_SIZE, d), gen, device, torch.bfloat16)
    v = _normal((total, Hkv, PAGE_SIZE, d), gen, device, torch.bfloat16)
    if nan_poison:
        _poison_paged_tails(k, v, lens, table)
    return dict(q=q, rho=rho, k_cache=k, v_cache=v,
                page_table=torch.from_numpy(table).to(device),
                cu_seqlens_q=torch.from_numpy(cu).to(device),
                seq_lens=torch.from_numpy(lens).to(device),
                q_lens=q_lens.astype(np.int64), seq_lens_host=lens.astype(np.int64),
                max_q_len=int(q_lens.max(initial=0)), scale=w.scale, causal=w.causal)


def small_chunked_prefill_inputs(q_lens, prefix_lens, num_heads, num_kv_heads, head_dim=128, *,
                                 rho_scale=0.1, seed=0, device="cpu"):
    """Chunked prefill inputs of arbitrary (small) shape; every pool slot
    outside a sequence is NaN."""
    cu, lens, table, total = chunked_layout(q_lens, prefix_lens, seed + 1)
    gen = _gen("cpu", seed)
    H, Hkv, d = num_heads, num_kv_heads, head_dim
    tq = int(cu[-1])
    q = torch.randn((tq, H, d), generator=gen).to(torch.bfloat16)
    rho = (torch.randn((tq, H, d), generator=gen) * rho_scale).to(torch.bfloat16)
    k = torch.full((total, Hkv, PAGE_SIZE, d), float("nan"), dtype=torch.bfloat16)
    v = torch.full((total, Hkv, PAGE_SIZE, d), float("nan"), dtype=torch.bfloat16)
    for b, n in enumerate(lens):
        for j in range(-(-int(n) // PAGE_SIZE)):
            take = min(PAGE_SIZE, int(n) - j * PAGE_SIZE)
            k[table[b, j], :, :take] = torch.randn((Hkv, take, d), generator=gen).to(torch.bfloat16)
            v[table[b, j], :, :take] = torch.randn((Hkv, take, d), generator=gen).to(torch.bfloat16)
    res = dict(q=q, rho=rho, k_cache=k, v_cache=v, page_table=torch.from_numpy(table),
               cu_seqlens_q=torch.from_numpy(cu), seq_lens=torch.from_numpy(lens),
               q_lens=np.asarray(q_lens, dtype=np.int64), seq_lens_host=lens.astype(np.int64),
               max_q_len=int(max(q_lens, default=0)), scale=1.0 / math.sqrt(d), causal=True)
    if device != "cpu":
        res = {kk: (vv.to(device) if torch.is_tensor(vv) else vv) for kk, vv in res.items()}
    return res


def chunked_prefill_flops(q_lens, seq_lens, num_heads, head_dim, causal=True) -> int:
    """Algorithmic FLOP of one chunked prefill call: 8*d per visible
    (query, key) pair.  Query i of a chunk of q rows over L keys sees
    L - q + i + 1 keys (causal) or L."""
    total = 0
    for q, L in zip(q_lens, seq_lens):
        q, L = int(q), int(L)
        total += q * (L - q) + q * (q + 1) // 2 if causal else q * L
    return 8 * head_dim * num_heads * total


def dout_like(q, seed):
    """dL/dout of a prefill: N(0, 1) draws rounded to bfloat16, shaped like q,
    on q's device (a generator of its own, so q, rho, k, v are unchanged)."""
    gen = _gen(q.device, seed)
    return _normal(tuple(q.shape), gen, q.device, torch.bfloat16)


def prefill_backward_flops(w: PrefillWorkload) -> int:
    """Algorithmic FLOP of one prefill backward: 16*d per visible pair, one
    pass over each product the gradients need (S, A, D = g.v, dQ, dR, dV and
    the two dK products, 2*d each)."""
    return 2 * prefill_flops(w)


def lla_decode_flops(w: DecodeWorkload, seq_lens=None) -> int:
    """Algorithmic FLOP of one LLA decode call: per (sequence, query head)
    with n keys, the scores (2*d*n), the two d x d weighted sums
    sum e k k^T and sum e k v^T (2 * 2*d*d*n), the first moments (2 * 2*d*n),
    the Cholesky factorisation and two triangular solves (d^3/3 + 2*d^2)
    and the output's matrix-vector product (2*d*d)."""
    d = w.head_dim
    lens = [w.kv_len] * w.batch if seq_lens is None else [int(x) for x in seq_lens]
    per_key = 2 * d + 4 * d * d + 4 * d
    per_head = d ** 3 // 3 + 4 * d * d
    return sum(w.num_q_heads * (n * per_key + (per_head if n else 0)) for n in lens)

