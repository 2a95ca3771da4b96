"""The prepared decode (parallax_decode_plan_*) against the one-shot call.

A plan made from fixed buffers must give, at every run, bit for bit what
parallax_decode gives on the buffers' current contents: it reuses the
validated arguments and tensor maps, not any data.  parallax_decode itself is
checked against the float64 oracle in test_decode_gpu.py; one case here is
checked against the oracle directly as well.
"""

import pytest
import torch

from parallax_local_linear_b200 import workloads as W
from tests.helpers import TOL_BF16, assert_parity, oracle_heads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def px():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from parallax_local_linear_b200 import binding
    return binding


def _cuda(inp):
    return {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}


CASES = {
    "cluster_grid": dict(args=(8, 16, 8, 128, 4096), kw={}, ctas=0),
    "workspace_merge": dict(args=(4, 8, 2, 128, 3000), kw=dict(seq_lens=[3000, 1200, 65, 0]), ctas=5),
    "paged": dict(args=(3, 16, 4, 128, 2500), kw=dict(seq_lens=[2500, 700, 64], paged=True), ctas=7),
    "f32": dict(args=(2, 4, 2, 64, 1000), kw=dict(dtype="f32"), ctas=3),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_plan_runs_match_the_one_shot_call(px, case):
    c = CASES[case]
    inp = _cuda(W.small_decode_inputs(*c["args"], seed=61, **c["kw"]))
    out = torch.empty_like(inp["q"])
    plan = px.DecodePlan(inp["q"], inp["rho"], inp["k_cache"], inp["v_cache"], inp["scale"], out=out,
                         seq_lens=inp.get("seq_lens"), page_table=inp.get("page_table"), num_ctas=c["ctas"])
    for step in range(3):
        if step == 2:   # new contents in the same buffers: the plan reads them at the run
            inp["q"].copy_(torch.randn_like(inp["q"].float()).to(inp["q"].dtype))
        plan.run()
        ref = px.decode(inp["q"], inp["rho"], inp["k_cache"], inp["v_cache"], inp["scale"],
                        seq_lens=inp.get("seq_lens"), page_table=inp.get("page_table"), num_ctas=c["ctas"])
        assert torch.equal(out, ref), f"{case} step {step}"
    assert px.last_device_error() == 0


def test_plan_against_the_oracle(px):
    inp = _cuda(W.small_decode_inputs(2, 8, 2, 128, 777, seed=62))
    out = torch.empty(inp["q"].shape, dtype=torch.bfloat16, device="cuda")
    plan = px.DecodePlan(inp["q"], inp["rho"], inp["k_cache"], inp["v_cache"], inp["scale"], out=out)
    plan.run()
    ref = oracle_heads(inp, [(b, h) for b in range(2) for h in range(8)])
    assert_parity(out.float().cpu().numpy(), ref, TOL_BF16, "plan")


def test_plan_in_a_cuda_graph(px):
    inp = _cuda(W.small_decode_inputs(4, 8, 4, 128, 2048, seed=63))
    out = torch.empty_like(inp["q"])
    plan = px.DecodePlan(inp["q"], inp["rho"], inp["k_cache"], inp["v_cache"], inp["scale"], out=out)
    plan.run()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        plan.run()
    out.zero_()
    g.replay()
    ref = px.decode(inp["q"], inp["rho"], inp["k_cache"], inp["v_cache"], inp["scale"])
    assert torch.equal(out, ref)


def test_plan_step_from_host_memory(px):
    # run_io: q and rho read by the kernel from pinned host memory, the
    # decode, the output written straight into pinned host memory: the result
    # equals the device-side run.
    inp = _cuda(W.small_decode_inputs(8, 16, 8, 128, 1024, seed=64))
    dq, dr = torch.empty_like(inp["q"]), torch.empty_like(inp["rho"])
    out = torch.empty_like(inp["q"])
    plan = px.DecodePlan(dq, dr, inp["k_cache"], inp["v_cache"], inp["scale"], out=out)
    hq, hr = inp["q"].cpu().pin_memory(), inp["rho"].cpu().pin_memory()
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    plan.run_io(hq, hr, hout)
    torch.cuda.synchronize()
    ref = px.decode(inp["q"], inp["rho"], inp["k_cache"], inp["v_cache"], inp["scale"])
    assert torch.equal(hout, ref.cpu())
    # a pageable buffer takes the copy path through the plan's buffers
    hout2 = torch.zeros(out.shape, dtype=out.dtype)
    plan.run_io(inp["q"].cpu(), inp["rho"].cpu(), hout2)
    torch.cuda.synchronize()
    assert torch.equal(hout2, ref.cpu())
    assert torch.equal(out.cpu(), ref.cpu())
    with pytest.raises(ValueError):
        plan.run_io(inp["q"], hr, hout)   # a device tensor where a host one belongs


def test_host_steps_chained_without_synchronisation(px):
    # Zero-copy run_io steps back to back on one stream: each launch reads its
    # q and rho from pinned host memory as it starts (possibly while the
    # previous step still runs), and its K and V only after the previous
    # kernel has finished.  Between two steps the cache is rescaled by a
    # device op on the same stream: the second step must see the new cache.
    inp = _cuda(W.small_decode_inputs(8, 16, 8, 128, 2048, seed=65))
    out = torch.empty_like(inp["q"])
    plan = px.DecodePlan(torch.empty_like(inp["q"]), torch.empty_like(inp["rho"]), inp["k_cache"], inp["v_cache"],
                         inp["scale"], out=out)
    gen = torch.Generator().manual_seed(7)
    steps = []
    for i in range(4):
        hq = (torch.randn(inp["q"].shape, generator=gen)).to(inp["q"].dtype).pin_memory()
        hr = (0.1 * torch.randn(inp["rho"].shape, generator=gen)).to(inp["rho"].dtype).pin_memory()
        hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        steps.append((hq, hr, hout))
    v0 = inp["v_cache"].clone()
    for i, (hq, hr, hout) in enumerate(steps):
        plan.run_io(hq, hr, hout)
        if i == 1:
            inp["v_cache"].mul_(2.0)   # exact in bf16: the later steps' outputs double
    torch.cuda.synchronize()
    for i, (hq, hr, hout) in enumerate(steps):
        v = inp["v_cache"] if i >= 2 else v0
        ref = px.decode(hq.cuda(), hr.cuda(), inp["k_cache"], v, inp["scale"])
        assert torch.equal(hout, ref.cpu()), f"step {i}"
