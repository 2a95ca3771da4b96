"""GPU parity of the chunked (append) prefill over the paged cache.

Sequence b holds L_b keys in 64-token pages placed by a seeded permutation;
its chunk of q_len_b queries are its last positions.  Rows of the CUDA
output are compared with the float64 oracle's explicit definition over the
keys each query sees, on the same seeded inputs:
    max |gpu - ref| <= 2e-2 * (1 + |ref|)   (bf16 inputs, fp32 accumulation).
Every pool slot outside a sequence is NaN, so an over-read of K or V shows
up as a non-finite output.  Chunks cover one row, partial and full 128-row
query tiles, ragged prefixes that put the causal diagonal anywhere inside a
64-key page, empty chunks, and the full 8-sequence workload on sampled rows.
"""

import numpy as np
import pytest
import torch

import oracle
from parallax_local_linear_b200 import workloads as W
from tests.helpers import TOL_BF16, F64View, assert_parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def px():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from parallax_local_linear_b200 import binding
    return binding


def _inputs(q_lens, prefix, H=2, Hkv=1, seed=0, rho_scale=0.1):
    return W.small_chunked_prefill_inputs(q_lens, prefix, H, Hkv, 128, rho_scale=rho_scale, seed=seed,
                                          device="cuda")


def _run(px, x, causal=True, out_dtype=torch.float32, out=None):
    return px.prefill_paged(x["q"], x["rho"], x["k_cache"], x["v_cache"], x["page_table"], x["cu_seqlens_q"],
                            x["seq_lens"], max_q_len=x["max_q_len"], scale=x["scale"], causal=causal,
                            out=out, out_dtype=out_dtype)


def _rows(x, H, limit=None, seed=0):
    rows = [(b, i, h) for b, m in enumerate(x["q_lens"]) for i in range(int(m)) for h in range(H)]
    if limit is not None and len(rows) > limit:
        rng = np.random.default_rng(seed)
        keep = set(rng.choice(len(rows), size=limit, replace=False).tolist())
        edges = {(b, i, h) for b, m in enumerate(x["q_lens"]) for h in range(H)
                 for i in (0, 1, int(m) - 1, 127, 128) if 0 <= i < int(m)}
        rows = sorted(edges | {rows[j] for j in keep})
    return rows


def _ref(x, rows, causal=True):
    v = {k: F64View(x[k]) for k in ("q", "rho", "k_cache", "v_cache")}
    return oracle.prefill_paged_rows(v["q"], v["rho"], v["k_cache"], v["v_cache"], x["page_table"].cpu().numpy(),
                                     x["cu_seqlens_q"].cpu().numpy(), x["seq_lens_host"], rows, x["scale"],
                                     causal=causal)


def _got(x, out, rows):
    cu = x["cu_seqlens_q"].cpu().numpy()
    o = out.float().cpu().numpy()
    return np.stack([o[cu[b] + i, h] for b, i, h in rows])


CASES = {
    "mixed": ([1, 63, 128, 129, 300], [0, 5, 64, 1000, 77]),
    "no_prefix": ([700], [0]),
    "long_prefix": ([200, 3], [130, 4000]),
    "diagonal_offsets": ([130, 130, 130, 130], [1, 31, 63, 65]),
    "with_empty_chunks": ([0, 90, 0], [40, 10, 0]),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_chunks_against_oracle(px, name):
    q_lens, prefix = CASES[name]
    x = _inputs(q_lens, prefix, seed=len(name))
    out = _run(px, x)
    rows = _rows(x, 2, limit=200, seed=1)
    assert_parity(_got(x, out, rows), _ref(x, rows), TOL_BF16, name)
    assert px.last_device_error() == 0


def test_non_causal(px):
    x = _inputs([50, 200], [100, 7], seed=3)
    out = _run(px, x, causal=False)
    rows = _rows(x, 2, limit=150)
    assert_parity(_got(x, out, rows), _ref(x, rows, causal=False), TOL_BF16, "non-causal")


def test_gqa_and_unit_probe(px):
    x = _inputs([150, 257], [33, 500], H=8, Hkv=2, seed=5, rho_scale=1.0)
    out = _run(px, x, out_dtype=torch.bfloat16)
    assert out.dtype == torch.bfloat16
    rows = _rows(x, 8, limit=200)
    assert_parity(_got(x, out, rows), _ref(x, rows), TOL_BF16, "gqa, unit rho, bf16 out")


def test_chunk_without_prefix_equals_dense_prefill(px):
    # A chunk with no cached prefix is a plain causal prefill: same tiles, same
    # arithmetic, keys read through the page table instead of a dense row.
    T = 1000
    x = _inputs([T], [0], seed=7)
    table = x["page_table"].cpu().numpy()[0]
    k = torch.stack([x["k_cache"][int(table[j])] for j in range(-(-T // 64))], 0)   # [pages, Hkv, 64, d]
    v = torch.stack([x["v_cache"][int(table[j])] for j in range(-(-T // 64))], 0)
    kd = k.permute(1, 0, 2, 3).reshape(1, -1, 64 * k.shape[0], 128)[:, :, :T].contiguous()
    vd = v.permute(1, 0, 2, 3).reshape(1, -1, 64 * v.shape[0], 128)[:, :, :T].contiguous()
    qd = x["q"].permute(1, 0, 2)[None].contiguous()
    rd = x["rho"].permute(1, 0, 2)[None].contiguous()
    dense = px.prefill(qd, rd, kd, vd, causal=True, scale=x["scale"], out_dtype=torch.float32)
    paged = _run(px, x)
    assert torch.equal(paged.permute(1, 0, 2)[None], dense)


def test_chunked_rows_match_one_prefill(px):
    # Appending [600, 1000) to a 600-token prefix gives the rows a single
    # causal prefill of all 1000 tokens gives at those positions.
    T, P0 = 1000, 600
    full = _inputs([T], [0], seed=9)
    whole = _run(px, full)
    chunk = dict(full)
    chunk["q"] = full["q"][P0:].contiguous()
    chunk["rho"] = full["rho"][P0:].contiguous()
    chunk["cu_seqlens_q"] = torch.tensor([0, T - P0], dtype=torch.int32, device="cuda")
    chunk["q_lens"] = np.array([T - P0])
    chunk["max_q_len"] = T - P0
    part = _run(px, chunk)
    np.testing.assert_allclose(part.cpu().numpy(), whole[P0:].cpu().numpy(), rtol=0, atol=2e-3)


def test_one_token_chunks_match_decode(px):
    x = _inputs([1, 1, 1, 1], [0, 63, 64, 3000], H=4, Hkv=2, seed=11)
    out = _run(px, x)
    q = x["q"].contiguous()
    dec = px.decode(q, x["rho"], x["k_cache"], x["v_cache"], x["scale"], seq_lens=x["seq_lens"],
                    page_table=x["page_table"], out_dtype=torch.float32)
    np.testing.assert_allclose(out.cpu().numpy(), dec.cpu().numpy(), rtol=0, atol=2e-2)


def test_rows_outside_every_sequence_are_untouched(px):
    x = _inputs([70, 5], [10, 200], seed=13)
    extra = 40
    for key in ("q", "rho"):
        pad = torch.zeros((extra,) + tuple(x[key].shape[1:]), dtype=x[key].dtype, device="cuda")
        x[key] = torch.cat([x[key], pad]).contiguous()
    out = torch.full(x["q"].shape, 123.0, dtype=torch.float32, device="cuda")
    _run(px, x, out=out)
    assert torch.all(out[-extra:] == 123.0)
    assert torch.isfinite(out[:-extra]).all()


def test_no_queries_is_a_no_op(px):
    x = _inputs([0, 0], [5, 70], seed=15)
    out = torch.empty((0, 2, 128), dtype=torch.float32, device="cuda")
    px.prefill_paged(x["q"], x["rho"], x["k_cache"], x["v_cache"], x["page_table"], x["cu_seqlens_q"],
                     x["seq_lens"], max_q_len=0, scale=x["scale"], out=out)
    assert px.last_device_error() == 0


def test_bad_page_sets_error_word_and_skips_the_sequence(px):
    x = _inputs([64, 64], [100, 0], seed=17)
    table = x["page_table"].clone()
    table[0, 1] = x["k_cache"].shape[0]          # one past the pool
    x["page_table"] = table
    out = torch.full(x["q"].shape, 7.0, dtype=torch.float32, device="cuda")
    _run(px, x, out=out)
    assert px.last_device_error() == px.DEVERR_BAD_PAGE
    assert torch.all(out[:64] == 7.0)
    rows = [(1, i, h) for i in (0, 63) for h in range(2)]
    assert_parity(_got(x, out, rows), _ref(x, rows), TOL_BF16, "good sequence")


@pytest.mark.parametrize("fault", ["chunk_longer_than_sequence", "chunk_above_max_q_len", "beyond_pages"])
def test_bad_lengths_set_error_word(px, fault):
    x = _inputs([64, 64], [100, 0], seed=19)
    if fault == "chunk_longer_than_sequence":
        x["seq_lens"] = torch.tensor([164, 10], dtype=torch.int32, device="cuda")
    elif fault == "chunk_above_max_q_len":
        x["max_q_len"] = 32
    else:
        x["seq_lens"] = torch.tensor([164, 64 * x["page_table"].shape[1] + 1], dtype=torch.int32, device="cuda")
    out = torch.full(x["q"].shape, 7.0, dtype=torch.float32, device="cuda")
    _run(px, x, out=out)
    assert px.last_device_error() == px.DEVERR_BAD_LENGTH
    assert torch.all(out[64:] == 7.0)


def test_full_chunked_workload_sampled(px):
    w = W.WORKLOADS["prefill_paged"]
    x = W.chunked_prefill_inputs(w, device="cuda")
    out = _run(px, x, out_dtype=torch.bfloat16)
    rng = np.random.default_rng(21)
    rows = [(0, 0, 0), (1, int(x["q_lens"][1]) - 1, 15), (4, 127, 3), (4, 128, 4)]
    rows += [(int(b), int(rng.integers(x["q_lens"][b])), int(rng.integers(16)))
             for b in rng.integers(0, w.batch, size=40)]
    assert_parity(_got(x, out, rows), _ref(x, rows), TOL_BF16, "chunked workload")
    assert torch.isfinite(out.float()).all()
    assert px.last_device_error() == 0
