"""A kernel wait that runs out of time is reported and leaves the device usable.

Every wait of one CTA role on another (a TMA load landing, tensor-core
results, a freed ring stage) is bounded by the device's pipeline wait limit.
These tests set that limit to 0, so the first wait that does not find its
phase complete gives up: the kernel must set PLX_DEVERR_TIMEOUT, wait for its
own copies and tensor-core operations in flight (those waits keep their own
long limit), free its tensor memory and return.  The next call with the
default limit, on the same stream and workspace, must then match the float64
oracle.  No GPU fault is involved: the failure is an ordinary bounded wait
that returns false.
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


def _timed_out(px, call):
    """Runs `call` with a zero wait limit; returns the error word it left."""
    assert px.last_device_error() == 0
    prev = px.set_wait_limit_ns(0)
    try:
        call()
        code = px.last_device_error()   # synchronises: the call has returned on the device
    finally:
        px.set_wait_limit_ns(prev)
    assert prev == 2_000_000_000
    return code


@pytest.mark.parametrize("ctas", [3, 0])
def test_decode_wait_timeout_then_recovery(px, ctas):
    # ctas 3: pieces merged through the workspace; 0: the unit-aligned grid
    # of 64 units on two CTAs each, whose clusters merge through distributed
    # shared memory.  Every CTA has more tiles than ring stages, so the
    # producer's first wait for a freed stage comes right after it has issued
    # the first loads, before any can have been consumed: with the zero limit
    # that wait gives up, whatever the timing.
    B, Hq, Hkv, L = (2, 4, 2, 8192) if ctas == 3 else (8, 16, 8, 4096)
    inp = W.small_decode_inputs(B, Hq, Hkv, 128, L, seed=51)
    inp = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    if ctas == 0:
        p = px.decode_params(inp["q"], inp["k_cache"])
        assert px.decode_num_ctas(p) == 2 * B * Hkv   # the clustered grid

    def run():
        return px.decode(inp["q"], inp["rho"], inp["k_cache"], inp["v_cache"], inp["scale"],
                         out_dtype=torch.float32, num_ctas=ctas)

    code = _timed_out(px, run)
    assert code & px.DEVERR_TIMEOUT, f"error word {code}"
    out = run()
    assert px.last_device_error() == 0
    heads = [(b, h) for b in range(B) for h in range(Hq)][:: max(1, B * Hq // 16)]
    ref = oracle_heads(inp, heads)   # [B, Hq, d], NaN outside `heads`
    got = np.stack([out[b, h].cpu().numpy() for b, h in heads])
    assert_parity(got, np.stack([ref[b, h] for b, h in heads]), TOL_BF16, f"decode after a timeout, ctas={ctas}")


def test_prefill_wait_timeout_then_recovery(px):
    inp = W.small_prefill_inputs(1, 2, 1000, 128, seed=52)
    inp = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}

    def run():
        return px.prefill(inp["q"], inp["rho"], inp["k"], inp["v"], causal=True, scale=inp["scale"],
                          out_dtype=torch.float32)

    code = _timed_out(px, run)
    assert code & px.DEVERR_TIMEOUT, f"error word {code}"
    out = run().cpu().numpy()
    assert px.last_device_error() == 0
    rows = [(0, h, t) for h in range(2) for t in (0, 1, 127, 128, 500, 999)]
    views = {k: F64View(inp[k]) for k in ("q", "rho", "k", "v")}
    ref = oracle.prefill_rows(views["q"], views["rho"], views["k"], views["v"], rows, inp["scale"])
    assert_parity(np.stack([out[b, h, t] for b, h, t in rows]), ref, TOL_BF16, "prefill after a timeout")


def test_backward_wait_timeout_then_recovery(px):
    x = W.small_prefill_inputs(1, 2, 300, 128, seed=53)
    x = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    dout = W.dout_like(x["q"], 54)
    out, vbar, stats = px.prefill_train(x["q"], x["rho"], x["k"], x["v"], True, x["scale"], out_dtype=torch.float32)

    def run():
        return px.prefill_backward(x["q"], x["rho"], x["k"], x["v"], out, vbar, stats, dout, True, x["scale"])

    code = _timed_out(px, run)
    assert code & px.DEVERR_TIMEOUT, f"error word {code}"
    grads = run()
    assert px.last_device_error() == 0
    ref = oracle.prefill_grads(*(to_f64(t) for t in (x["q"], x["rho"], x["k"], x["v"], dout)), x["scale"],
                               causal=True)
    for name, g, r in zip(("dq", "drho", "dk", "dv"), grads, ref):
        assert_parity(g.cpu().numpy(), r, TOL_BF16, f"{name} after a timeout")


def test_wait_limit_setter_round_trips(px):
    prev = px.set_wait_limit_ns(123456)
    try:
        assert px.set_wait_limit_ns(prev) == 123456
    finally:
        px.set_wait_limit_ns(prev)


@pytest.mark.parametrize("num_ctas", [0, 8])
def test_lla_wait_timeout_then_recovery(px, num_ctas):
    # num_ctas 0: heads cut into pieces, a moments grid and a solve grid; 8
    # (one CTA per head): one grid, the solve in place in the moments kernel.
    inp = W.small_decode_inputs(2, 4, 2, 128, 4096, seed=55)
    inp = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}

    def run():
        return px.lla_decode(inp["q"], inp["k_cache"], inp["v_cache"], inp["scale"], 0.01, out_dtype=torch.float32,
                             num_ctas=num_ctas)

    code = _timed_out(px, run)
    assert code & px.DEVERR_TIMEOUT, f"error word {code}"
    out, rho = run()
    assert px.last_device_error() == 0
    rho_ref, ref = oracle.lla_decode(to_f64(inp["q"]), F64View(inp["k_cache"]), F64View(inp["v_cache"]),
                                     inp["scale"], 0.01)
    assert_parity(out.cpu().numpy(), ref, TOL_BF16, "LLA after a timeout")
