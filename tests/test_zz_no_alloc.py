"""The decode entry point that allocates nothing (parallax_decode_noalloc).

Some callers cannot allocate device memory: a plugin inside an application
that budgets all GPU memory itself, a language binding without a CUDA
allocator, a latency-critical path that must not call cudaMalloc.  For them
the library keeps the split partials in its own fixed device array instead
of a caller workspace.  These tests call that entry point through the C ABI
and compare it with parallax_decode (which takes a workspace) on the same
inputs, twice in a row, since every call reuses the array the previous call
left behind.  The file sorts last so a stop-at-first-failure run has already
run every other test.
"""

import ctypes

import pytest
import torch

from parallax_local_linear_b200 import workloads as W
from tests.helpers import TOL_BF16, TOL_F32, assert_parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def px():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from parallax_local_linear_b200 import binding
    return binding


def _inputs(case):
    if case == "contiguous_bf16":
        inp = W.small_decode_inputs(4, 8, 2, 128, 3000, seq_lens=[3000, 1200, 65, 1], seed=31)
    elif case == "paged_bf16":
        inp = W.small_decode_inputs(3, 16, 4, 128, 2500, seq_lens=[2500, 700, 64], paged=True, seed=32)
    else:
        inp = W.small_decode_inputs(2, 4, 2, 64, 1000, dtype="f32", seed=33)
    return {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}


def _noalloc(px, inp, out, ctas):
    p = px.decode_params(inp["q"], inp["k_cache"], page_table=inp.get("page_table"), scale=inp["scale"],
                         out_dtype=out.dtype, num_ctas=ctas)
    return px.lib.parallax_decode_noalloc(
        px._ptr(inp["q"]), px._ptr(inp["rho"]), px._ptr(inp["k_cache"]), px._ptr(inp["v_cache"]),
        px._ptr(inp.get("page_table")), px._ptr(inp.get("seq_lens")), px._ptr(out), ctypes.byref(p),
        px._stream_ptr(inp["q"].device))


@pytest.mark.parametrize("case", ["contiguous_bf16", "paged_bf16", "f32"])
def test_noalloc_matches_workspace_entry_point(px, case):
    inp = _inputs(case)
    ctas = 5   # several CTAs per sequence, so the scratch array is in use
    ref = px.decode(inp["q"], inp["rho"], inp["k_cache"], inp["v_cache"], inp["scale"],
                    seq_lens=inp.get("seq_lens"), page_table=inp.get("page_table"),
                    out_dtype=torch.float32, num_ctas=ctas)
    tol = TOL_F32 if case == "f32" else TOL_BF16
    for call in range(2):
        out = torch.full_like(ref, float("nan"))
        assert _noalloc(px, inp, out, ctas) == 0
        torch.cuda.synchronize()
        assert_parity(out.cpu().numpy(), ref.cpu().numpy(), tol, f"{case} call {call}")
    assert px.last_device_error() == 0


@pytest.mark.parametrize("case", ["default_grid", "empty_sequence"])
def test_noalloc_default_grid_and_empty_sequences(px, case):
    # The default grid (num_ctas 0) of an equal-length contiguous cache is
    # unit-aligned and may merge a unit's pieces inside a thread-block
    # cluster; a zero-length sequence gets a zero output without any tile.
    if case == "default_grid":
        inp = W.small_decode_inputs(8, 16, 8, 128, 4096, seed=34)
    else:
        inp = W.small_decode_inputs(4, 8, 2, 128, 1500, seq_lens=[1500, 0, 700, 0], seed=35)
    inp = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    ref = px.decode(inp["q"], inp["rho"], inp["k_cache"], inp["v_cache"], inp["scale"],
                    seq_lens=inp.get("seq_lens"), out_dtype=torch.float32, num_ctas=0)
    for call in range(2):
        out = torch.full_like(ref, float("nan"))
        assert _noalloc(px, inp, out, 0) == 0
        torch.cuda.synchronize()
        assert_parity(out.cpu().numpy(), ref.cpu().numpy(), TOL_BF16, f"{case} call {call}")
    if case == "empty_sequence":
        assert torch.equal(out[1], torch.zeros_like(out[1])) and torch.equal(out[3], torch.zeros_like(out[3]))
    assert px.last_device_error() == 0


def test_noalloc_back_to_back_different_shapes(px):
    a, b = _inputs("contiguous_bf16"), _inputs("paged_bf16")
    for inp in (a, b, a):
        ref = px.decode(inp["q"], inp["rho"], inp["k_cache"], inp["v_cache"], inp["scale"],
                        seq_lens=inp.get("seq_lens"), page_table=inp.get("page_table"),
                        out_dtype=torch.float32, num_ctas=7)
        out = torch.empty_like(ref)
        assert _noalloc(px, inp, out, 7) == 0
        assert_parity(out.cpu().numpy(), ref.cpu().numpy(), TOL_BF16, "back to back")


def test_noalloc_rejects_what_does_not_fit(px):
    inp = _inputs("contiguous_bf16")
    p = px.decode_params(inp["q"], inp["k_cache"], num_ctas=40)
    big = px.DecodeParams(512, 64, 8, 128, 65536, 0, 0, 0, 1, 1, 0.088, 100000)
    assert px.decode_workspace_size(big) > px.NOALLOC_SCRATCH_BYTES
    out = torch.empty(1, device="cuda")
    st = px.lib.parallax_decode_noalloc(px._ptr(out), px._ptr(out), px._ptr(out), px._ptr(out), None, None,
                                        px._ptr(out), ctypes.byref(big), px._stream_ptr(out.device))
    assert st == 3   # PLX_ERR_WORKSPACE, before any launch
    assert px.decode_workspace_size(p) <= px.NOALLOC_SCRATCH_BYTES
