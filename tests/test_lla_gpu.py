"""GPU parity of Local Linear Attention with the solved probe (decode).

parallax_lla_decode is compared with the float64 oracle (oracle.lla_decode:
rho* = (S_KK + ridge I)^-1 (kbar - q) by numpy.linalg.solve, then
vbar - S_KV^T rho*) on the same seeded bf16 inputs, for the output and the
solved probe:  max |gpu - ref| <= 2e-2 * (1 + |ref|)  (bf16 inputs, fp32
accumulation and solve).  Inputs are well conditioned for the solve: many
more effectively weighted keys than the head dimension when ridge = 0, and
ridge > 0 for short sequences (the pages name no regularisation).
"""

import numpy as np
import pytest
import torch

import oracle
from parallax_local_linear_b200 import workloads as W
from tests.helpers import TOL_BF16, F64View, assert_parity, oracle_heads, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def px():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from parallax_local_linear_b200 import binding
    return binding


def _cuda(inp):
    return {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}


def _run(px, inp, ridge, **kw):
    return px.lla_decode(inp["q"], inp["k_cache"], inp["v_cache"], inp["scale"], ridge,
                         seq_lens=inp.get("seq_lens"), page_table=inp.get("page_table"), **kw)


def _oracle(inp, ridge, heads=None):
    lens = None if inp.get("seq_lens") is None else inp["seq_lens"].cpu().numpy()
    table = None if inp.get("page_table") is None else inp["page_table"].cpu().numpy()
    return oracle.lla_decode(to_f64(inp["q"]), F64View(inp["k_cache"]), F64View(inp["v_cache"]), inp["scale"],
                             ridge, seq_lens=lens, page_table=table, heads=heads)


def _check(px, inp, ridge, what, heads=None, **kw):
    out, rho = _run(px, inp, ridge, out_dtype=torch.float32, **kw)
    rref, oref = _oracle(inp, ridge, heads)
    o, r = out.cpu().numpy(), rho.cpu().numpy()
    if heads is not None:
        sel = tuple(np.array(heads).T)
        o, r, oref, rref = o[sel], r[sel], oref[sel], rref[sel]
    assert_parity(o, oref, TOL_BF16, f"out {what}")
    assert_parity(r, rref, TOL_BF16, f"rho* {what}")
    assert px.last_device_error() == 0
    return out, rho


@pytest.mark.parametrize("L", [1024, 4096])
@pytest.mark.parametrize("ridge", [0.0, 0.05])
def test_contiguous(px, L, ridge):
    inp = _cuda(W.small_decode_inputs(2, 4, 2, 128, L, seed=L + 7))
    _check(px, inp, ridge, f"L={L} ridge={ridge}")


@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (8, 2), (8, 1)])
def test_query_head_groups(px, Hq, Hkv):
    inp = _cuda(W.small_decode_inputs(2, Hq, Hkv, 128, 2000, seed=Hq * 10 + Hkv))
    _check(px, inp, 0.01, f"Hq={Hq} Hkv={Hkv}")


@pytest.mark.parametrize("L", [1, 2, 5, 63, 64, 65, 200, 700])
def test_short_sequences_with_ridge(px, L):
    # Few keys: S_KK has rank < d, the ridge makes the system definite and the
    # probe large along the directions the keys do not span; the lo part of
    # e o K keeps the products exact enough for that.
    inp = _cuda(W.small_decode_inputs(2, 4, 2, 128, L, seed=300 + L))
    _check(px, inp, 0.1, f"short L={L}")


@pytest.mark.parametrize("num_ctas", [0, 32])
def test_ragged_paged_and_empty(px, num_ctas):
    # num_ctas 0: several pieces per head, merged by the solve grid; 32 (one
    # CTA per head): one piece, solved in place by the moments kernel.
    lens = [3000, 1200, 65, 0]
    inp = _cuda(W.small_decode_inputs(4, 8, 2, 128, 3072, seq_lens=lens, paged=True, seed=41))
    out, rho = _check(px, inp, 0.1, f"paged ragged, num_ctas={num_ctas}", num_ctas=num_ctas)
    assert not out[3].any() and not rho[3].any()   # an empty sequence: out = 0, rho* = 0
    contig = {k: inp[k] for k in ("q", "scale", "seq_lens")}
    contig.update(k_cache=inp["k_contig"], v_cache=inp["v_contig"])
    out_c, rho_c = _run(px, contig, 0.1, out_dtype=torch.float32, num_ctas=num_ctas)
    assert torch.equal(out, out_c) and torch.equal(rho, rho_c)   # same keys, same pieces: same bits


@pytest.mark.parametrize("pieces", [1, 3, 16])
def test_pieces_merge(px, pieces):
    inp = _cuda(W.small_decode_inputs(1, 2, 1, 128, 6000, seq_lens=[5000], seed=44))
    _check(px, inp, 0.0, f"pieces={pieces}", num_ctas=2 * pieces)


def test_noncentred_keys(px):
    inp = _cuda(W.small_decode_inputs(2, 4, 2, 128, 3000, key_offset_std=0.5, value_offset=2.0, seed=45))
    _check(px, inp, 0.0, "offset keys")


def test_bf16_output_and_determinism(px):
    inp = _cuda(W.small_decode_inputs(2, 4, 2, 128, 1500, seed=46))
    a, ra = _run(px, inp, 0.02)
    b, rb = _run(px, inp, 0.02)
    assert a.dtype == torch.bfloat16 and torch.equal(a, b) and torch.equal(ra, rb)
    _, oref = _oracle(inp, 0.02)
    assert_parity(a.float().cpu().numpy(), oref, TOL_BF16, "bf16 out")


def test_single_key_without_ridge_is_reported_singular(px):
    # One key and ridge 0: S_KK = 0 exactly, the first pivot is 0.  The head
    # reports PLX_DEVERR_SINGULAR and falls back to rho* = 0, out = vbar = v.
    inp = _cuda(W.small_decode_inputs(1, 2, 1, 128, 1, seed=47))
    out, rho = _run(px, inp, 0.0, out_dtype=torch.float32)
    assert px.last_device_error() & px.DEVERR_SINGULAR
    assert not rho.any()
    np.testing.assert_array_equal(out[0].cpu().numpy(), inp["v_cache"][0, 0].float().cpu().numpy().repeat(2, 0))


def test_decode_bf16_workload(px):
    w = W.WORKLOADS["decode_bf16"]
    inp = W.decode_inputs(w, device="cuda")
    _check(px, inp, 0.0, "decode_bf16 workload")


def test_decode_long_workload_sampled(px):
    w = W.WORKLOADS["decode_long"]
    inp = W.decode_inputs(w, device="cuda")
    rng = np.random.default_rng(8)
    heads = sorted({(0, 0), (63, 31)} | {(int(rng.integers(64)), int(rng.integers(32))) for _ in range(14)})
    _check(px, inp, 0.0, "decode_long workload", heads=heads)
    del inp
    torch.cuda.empty_cache()


def test_decode_after_lla_is_unaffected(px):
    # LLA's scratch is not the decode's workspace: a decode whose units are
    # split over CTAs (merged through the workspace counters) right after an
    # LLA call must still match the oracle.
    inp = _cuda(W.small_decode_inputs(1, 2, 2, 128, 500, seed=48))
    _run(px, inp, 0.1)
    out = px.decode(inp["q"], inp["q"], inp["k_cache"], inp["v_cache"], inp["scale"], out_dtype=torch.float32)
    ref = oracle_heads(dict(inp, rho=inp["q"]), [(0, 0), (0, 1)])
    assert_parity(out.cpu().numpy(), ref, TOL_BF16, "decode after LLA")


def test_chained_calls_read_the_previous_output(px):
    # The moments and solve grids, and consecutive calls, are chained by a
    # programmatic dependency: a call whose q is the previous call's output
    # (written by its solve just before) must see that output.
    inp = _cuda(W.small_decode_inputs(4, 8, 4, 128, 2048, seed=91))
    out1, _ = px.lla_decode(inp["q"], inp["k_cache"], inp["v_cache"], inp["scale"], 0.05)
    out2, rho2 = px.lla_decode(out1, inp["k_cache"], inp["v_cache"], inp["scale"], 0.05)
    out3, _ = px.lla_decode(out2, inp["k_cache"], inp["v_cache"], inp["scale"], 0.05)
    torch.cuda.synchronize()
    ref1, _ = px.lla_decode(inp["q"], inp["k_cache"], inp["v_cache"], inp["scale"], 0.05)
    torch.cuda.synchronize()
    ref2, rref2 = px.lla_decode(ref1, inp["k_cache"], inp["v_cache"], inp["scale"], 0.05)
    torch.cuda.synchronize()
    ref3, _ = px.lla_decode(ref2, inp["k_cache"], inp["v_cache"], inp["scale"], 0.05)
    torch.cuda.synchronize()
    assert torch.equal(out1, ref1) and torch.equal(out2, ref2) and torch.equal(out3, ref3)
    assert torch.equal(rho2, rref2)
