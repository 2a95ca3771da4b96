"""GPU parity of Parallax decode against the float64 oracle.

Every case runs the CUDA path through the C ABI (the ctypes binding) and the
oracle on the same seeded inputs, and checks
    max |gpu - ref| <= tol * (1 + |ref|),  tol = 1e-5 (fp32), 2e-2 (bf16).
Shapes span several 64-token tiles, ragged tails, GQA groups and split
counts; the named workloads run at full size with sampled heads.
"""

import numpy as np
import pytest
import torch

from parallax_local_linear_b200 import workloads as W
from tests.helpers import TOL_BF16, TOL_F32, assert_parity, oracle_heads, parity_error

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def px():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from parallax_local_linear_b200 import binding
    return binding


def _to(inp, device=DEV):
    return {k: (v.to(device) if torch.is_tensor(v) else v) for k, v in inp.items()}


def _run(px, inp, **kw):
    return px.decode(inp["q"], inp["rho"], inp["k_cache"], inp["v_cache"], inp["scale"],
                     seq_lens=inp.get("seq_lens"), page_table=inp.get("page_table"), **kw)


def _all_heads(inp):
    B, Hq, _ = inp["q"].shape
    return [(b, h) for b in range(B) for h in range(Hq)]


def _check_no_device_error(px):
    assert px.last_device_error() == 0


# ----------------------------------------------------------------- workloads

def test_decode_f32_workload(px):
    w = W.WORKLOADS["decode_f32"]
    inp = W.decode_inputs(w, device=DEV)
    out = _run(px, inp)
    ref = oracle_heads(inp, _all_heads(inp))
    assert out.dtype == torch.float32
    assert_parity(out.cpu().numpy(), ref, TOL_F32, "decode_f32")
    _check_no_device_error(px)


def test_decode_bf16_workload(px):
    w = W.WORKLOADS["decode_bf16"]
    inp = W.decode_inputs(w, device=DEV)
    out = _run(px, inp)
    assert out.dtype == torch.bfloat16
    ref = oracle_heads(inp, _all_heads(inp))
    assert_parity(out.float().cpu().numpy(), ref, TOL_BF16, "decode_bf16")
    _check_no_device_error(px)


def test_decode_long_workload_sampled(px):
    # 64 (sequence, query head) pairs: every sequence's first and last
    # sequences, all four query heads of some KV heads, the rest seeded.
    w = W.WORKLOADS["decode_long"]
    inp = W.decode_inputs(w, device=DEV)
    out = _run(px, inp).float().cpu().numpy()
    rng = np.random.default_rng(3)
    heads = {(0, 0), (0, 31), (63, 0), (63, 31), (17, 4), (17, 5), (17, 6), (17, 7), (40, 28), (40, 29),
             (40, 30), (40, 31)}
    while len(heads) < 64:
        heads.add((int(rng.integers(w.batch)), int(rng.integers(w.num_q_heads))))
    heads = sorted(heads)
    ref = oracle_heads(inp, heads)
    for b, h in heads:
        assert_parity(out[b, h], ref[b, h], TOL_BF16, f"decode_long ({b},{h})")
    assert np.isfinite(out).all()
    _check_no_device_error(px)
    del inp
    torch.cuda.empty_cache()


def test_decode_paged_workload_sampled(px):
    # Every one of the 128 sequences at one query head (so the shortest, the
    # longest and every length residue mod the 64-token page that the seed
    # draws are covered), plus all 16 heads of the shortest and the longest.
    w = W.WORKLOADS["decode_paged"]
    inp = W.decode_inputs(w, device=DEV)
    out = _run(px, inp).float().cpu().numpy()
    lens = inp["seq_lens"].cpu().numpy()
    b_short, b_long = int(np.argmin(lens)), int(np.argmax(lens))
    heads = {(b, b % w.num_q_heads) for b in range(w.batch)}
    heads |= {(b, h) for b in (b_short, b_long) for h in range(w.num_q_heads)}
    heads = sorted(heads)
    assert len({int(n) % 64 for n in lens}) > 32   # many page-boundary residues
    ref = oracle_heads(inp, heads)
    for b, h in heads:
        assert_parity(out[b, h], ref[b, h], TOL_BF16, f"decode_paged ({b},{h}) len={lens[b]}")
    assert np.isfinite(out).all()
    _check_no_device_error(px)
    del inp
    torch.cuda.empty_cache()


# ------------------------------------------------------------------- sweeps

@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("L", [1, 2, 63, 64, 65, 200, 1000, 4097])
@pytest.mark.parametrize("group", [1, 2, 4, 8])
def test_bf16_shapes(px, d, L, group):
    inp = _to(W.small_decode_inputs(2, 2 * group, 2, d, L, seed=L * 10 + group))
    out = _run(px, inp, out_dtype=torch.float32)
    ref = oracle_heads(inp, _all_heads(inp))
    assert_parity(out.cpu().numpy(), ref, TOL_BF16, f"d={d} L={L} g={group}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("L", [1, 31, 64, 65, 257, 1000])
@pytest.mark.parametrize("group", [1, 3])
def test_f32_shapes(px, d, L, group):
    inp = _to(W.small_decode_inputs(2, 2 * group, 2, d, L, dtype="f32", seed=L + group))
    out = _run(px, inp)
    ref = oracle_heads(inp, _all_heads(inp))
    assert_parity(out.cpu().numpy(), ref, TOL_F32, f"f32 d={d} L={L} g={group}")


@pytest.mark.parametrize("ctas", [1, 2, 3, 16, 0, 1000])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_grid_sizes_agree(px, ctas, dtype):
    # Different persistent grids cut the units into different pieces.
    inp = _to(W.small_decode_inputs(3, 8, 2, 128, 1500, dtype=dtype, seq_lens=[1500, 700, 65], seed=5))
    out = _run(px, inp, num_ctas=ctas, out_dtype=torch.float32)
    ref = oracle_heads(inp, _all_heads(inp))
    assert_parity(out.cpu().numpy(), ref, TOL_F32 if dtype == "f32" else TOL_BF16, f"ctas={ctas}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_ragged_lengths_with_nan_tails(px, dtype):
    lens = [1, 63, 64, 65, 128, 129, 700, 0]
    inp = _to(W.small_decode_inputs(8, 4, 2, 128, 768, dtype=dtype, seq_lens=lens, seed=11))
    out = _run(px, inp, out_dtype=torch.float32).cpu().numpy()
    ref = oracle_heads(inp, _all_heads(inp))
    assert np.isfinite(out).all(), "a NaN row past a sequence end leaked into the output"
    assert_parity(out, ref, TOL_F32 if dtype == "f32" else TOL_BF16, "ragged")
    np.testing.assert_array_equal(out[7], 0.0)   # empty sequence -> zero output


@pytest.mark.parametrize("ctas", [1, 4, 0])
def test_paged_is_bit_identical_to_contiguous(px, ctas):
    lens = [300, 64, 1, 129]
    inp = _to(W.small_decode_inputs(4, 8, 2, 128, 320, seq_lens=lens, paged=True, seed=3))
    paged = _run(px, inp, num_ctas=ctas, out_dtype=torch.float32)
    contig = px.decode(inp["q"], inp["rho"], inp["k_contig"], inp["v_contig"], inp["scale"],
                       seq_lens=inp["seq_lens"], num_ctas=ctas, out_dtype=torch.float32)
    assert torch.equal(paged, contig)
    ref = oracle_heads(inp, _all_heads(inp))
    assert_parity(paged.cpu().numpy(), ref, TOL_BF16, "paged")


def test_noncentred_keys_and_values(px):
    # Keys share a large offset per KV head (the output is invariant to it)
    # and values a common shift; the a_ref shift keeps the products small.
    inp = _to(W.small_decode_inputs(2, 8, 2, 128, 2000, key_offset_std=4.0, value_offset=3.0, seed=9))
    out = _run(px, inp, out_dtype=torch.float32)
    ref = oracle_heads(inp, _all_heads(inp))
    assert_parity(out.cpu().numpy(), ref, TOL_BF16, "non-centred")


def test_rho_zero_matches_softmax_attention_reference(px):
    inp = _to(W.small_decode_inputs(2, 4, 2, 128, 777, seed=21))
    inp["rho"] = torch.zeros_like(inp["rho"])
    out = _run(px, inp, out_dtype=torch.float32)
    ref = oracle_heads(inp, _all_heads(inp))
    assert_parity(out.cpu().numpy(), ref, TOL_BF16, "rho=0")


def test_output_guard_bands_untouched(px):
    inp = _to(W.small_decode_inputs(2, 4, 2, 128, 500, seed=4))
    n = inp["q"].numel()
    buf = torch.full((n + 2048,), 12345.0, dtype=torch.float32, device=DEV)
    out = buf[1024:1024 + n].view(inp["q"].shape)
    _run(px, inp, out=out, out_dtype=torch.float32, num_ctas=3)
    torch.cuda.synchronize()
    assert (buf[:1024] == 12345.0).all() and (buf[1024 + n:] == 12345.0).all()


def test_repeated_calls_are_deterministic(px):
    inp = _to(W.small_decode_inputs(4, 8, 2, 128, 3000, seed=8))
    a = _run(px, inp, num_ctas=7)
    b = _run(px, inp, num_ctas=7)
    assert torch.equal(a, b)


# ------------------------------------------------------------ device errors

def test_bad_page_id_sets_error_word(px):
    inp = _to(W.small_decode_inputs(2, 4, 2, 128, 200, seq_lens=[200, 100], paged=True, seed=6))
    assert px.last_device_error() == 0
    table = inp["page_table"].clone()
    table[1, 0] = 10 ** 6
    px.decode(inp["q"], inp["rho"], inp["k_cache"], inp["v_cache"], inp["scale"],
              seq_lens=inp["seq_lens"], page_table=table)
    assert px.last_device_error() & px.DEVERR_BAD_PAGE
    assert px.last_device_error() == 0   # reading clears it


def test_bad_length_sets_error_word(px):
    inp = _to(W.small_decode_inputs(2, 4, 2, 128, 200, seed=6))
    lens = torch.tensor([200, 500], dtype=torch.int32, device=DEV)
    px.decode(inp["q"], inp["rho"], inp["k_cache"], inp["v_cache"], inp["scale"], seq_lens=lens)
    assert px.last_device_error() & px.DEVERR_BAD_LENGTH


def test_workspace_too_small_is_rejected(px):
    import ctypes
    inp = _to(W.small_decode_inputs(2, 4, 2, 128, 2000, seed=1))
    p = px.decode_params(inp["q"], inp["k_cache"], num_ctas=4)
    need = px.decode_workspace_size(p)
    assert need > 0
    ws = torch.zeros(need - 256, dtype=torch.uint8, device=DEV)
    out = torch.empty_like(inp["q"])
    st = px.lib.parallax_decode(px._ptr(inp["q"]), px._ptr(inp["rho"]), px._ptr(inp["k_cache"]),
                                px._ptr(inp["v_cache"]), None, None, px._ptr(out), px._ptr(ws),
                                ws.numel(), ctypes.byref(p), px._stream_ptr(inp["q"].device))
    assert st == 3


@pytest.mark.parametrize("L", [2, 3, 5, 9])
@pytest.mark.parametrize("group", [2, 8])
def test_short_sequences_keep_near_fp32_accuracy(px, L, group):
    # With a handful of keys nothing averages out: the probe products e*a reach
    # ~10 and must enter the value product without bf16 rounding.
    inp = _to(W.small_decode_inputs(4, 2 * group, 2, 128, L, seed=100 + L))
    out = _run(px, inp, out_dtype=torch.float32)
    ref = oracle_heads(inp, _all_heads(inp))
    assert_parity(out.cpu().numpy(), ref, 2e-3, f"short L={L} g={group}")


@pytest.mark.parametrize("d", [64, 128])
def test_long_chunks_let_warps_run_ahead(px, d):
    # Few units and long sequences: every CTA streams tens of tiles, so its
    # consumer warps can drift a full ring apart (the stage / warp ownership
    # rule of the pipeline is what keeps their barrier waits exact).
    inp = _to(W.small_decode_inputs(1, 4, 1, d, 60000, seed=77))
    out = _run(px, inp, out_dtype=torch.float32, num_ctas=16)
    ref = oracle_heads(inp, _all_heads(inp))
    assert_parity(out.cpu().numpy(), ref, TOL_BF16, f"long chunks d={d}")
    assert px.last_device_error() == 0


@pytest.mark.parametrize("B,Hq,Hkv,L", [(8, 16, 8, 4096), (6, 32, 8, 1000), (4, 8, 2, 129), (16, 32, 8, 300)])
def test_unit_aligned_grid_and_cluster_merge(px, B, Hq, Hkv, L):
    # Equal-length contiguous caches run on a grid of k CTAs per (sequence,
    # KV head); for k = 2 or 3 each unit is one thread-block cluster that
    # merges its pieces through distributed shared memory.
    import ctypes
    inp = _to(W.small_decode_inputs(B, Hq, Hkv, 128, L, seed=B * 1000 + L))
    p = px.decode_params(inp["q"], inp["k_cache"])
    ctas = px.decode_num_ctas(p)
    units = B * Hkv
    assert ctas % units == 0 or ctas == min(148, units * (-(-L // 64)))
    out = _run(px, inp, out_dtype=torch.float32)
    ref = oracle_heads(inp, _all_heads(inp))
    assert_parity(out.cpu().numpy(), ref, TOL_BF16, f"aligned B={B} Hkv={Hkv} L={L} ctas={ctas}")
    again = _run(px, inp, out_dtype=torch.float32)
    assert torch.equal(out, again)
    assert px.last_device_error() == 0


@pytest.mark.parametrize("paged", [False, True])
def test_chained_calls_read_the_previous_output(px, paged):
    # Consecutive decodes on one stream are launched with a programmatic
    # dependency: the second may start before the first ends, and must wait
    # for it before reading its inputs.  Here the second call's q and rho are
    # the first call's output, written by the kernel just before; the chain
    # runs with no host synchronisation in between and must equal the same
    # two calls separated by a device synchronisation.
    inp = _to(W.small_decode_inputs(8, 16, 8, 128, 2048, dtype="bf16", paged=paged, seed=81))
    inp2 = _to(W.small_decode_inputs(8, 16, 8, 128, 2048, dtype="bf16", paged=paged, seed=82))
    kw = dict(seq_lens=inp2.get("seq_lens"), page_table=inp2.get("page_table"))
    out1 = _run(px, inp)
    out2 = px.decode(out1, out1, inp2["k_cache"], inp2["v_cache"], inp2["scale"], **kw)
    out3 = torch.empty_like(out2)
    for _ in range(3):   # a few more links, still without synchronising
        px.decode(out2, out1, inp2["k_cache"], inp2["v_cache"], inp2["scale"], out=out3, **kw)
        px.decode(out3, out1, inp2["k_cache"], inp2["v_cache"], inp2["scale"], out=out2, **kw)
    torch.cuda.synchronize()
    ref1 = _run(px, inp)
    torch.cuda.synchronize()
    ref2 = px.decode(ref1, ref1, inp2["k_cache"], inp2["v_cache"], inp2["scale"], **kw)
    torch.cuda.synchronize()
    for _ in range(3):
        ref3 = px.decode(ref2, ref1, inp2["k_cache"], inp2["v_cache"], inp2["scale"], **kw)
        torch.cuda.synchronize()
        ref2 = px.decode(ref3, ref1, inp2["k_cache"], inp2["v_cache"], inp2["scale"], **kw)
        torch.cuda.synchronize()
    assert torch.equal(out1, ref1)
    assert torch.equal(out2, ref2)
