"""GPU parity of the projected decode (q and rho projected from the layer
input in the same call) against the float64 oracle.

The projections are compared with the oracle's bfloat16 roundings of the
exact sums.  The kernel rounds an fp32 sum instead, which differs from the
exact one by at most hidden * 2^-23 * sum_c |x_c w_c| (recursive fp32
summation, with a factor 2 of slack for the tensor cores' accumulation); so
every element must be within that plus one bfloat16 spacing of the oracle's,
and almost all must be equal.  (Near zero the fp32 error can span several of
the tiny bfloat16 spacings there.)  The outputs are compared as in the plain
decode: max |gpu - ref| <= 2e-2 (1 + |ref|).  The programmatic dependency between the
two launches is checked by running the decode on projection buffers that
hold NaN beforehand, back to back and inside a CUDA graph.
"""

import numpy as np
import pytest
import torch

import oracle
from parallax_local_linear_b200 import workloads as W
from tests.helpers import TOL_BF16, F64View, assert_parity, to_f64

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


def _inputs(B, Hq, Hkv, d, L, hidden, seed, **kw):
    inp = _to(W.small_decode_inputs(B, Hq, Hkv, d, L, seed=seed, **kw))
    inp.update(W.projection_inputs(B, Hq, d, hidden, device=DEV, seed=seed + 1))
    return inp


def _run(px, inp, **kw):
    return px.decode_projected(inp["x"], inp["w_q"], inp["w_rho"], inp["k_cache"], inp["v_cache"], inp["scale"],
                               seq_lens=inp.get("seq_lens"), page_table=inp.get("page_table"), **kw)


def _oracle(inp, heads=None):
    lens = None if inp.get("seq_lens") is None else inp["seq_lens"].cpu().numpy()
    table = None if inp.get("page_table") is None else inp["page_table"].cpu().numpy()
    return oracle.decode_projected(to_f64(inp["x"]), to_f64(inp["w_q"]), to_f64(inp["w_rho"]),
                                   F64View(inp["k_cache"]), F64View(inp["v_cache"]), inp["scale"],
                                   seq_lens=lens, page_table=table, heads=heads)


def _bf16_spacing(x):
    _, e = np.frexp(x)
    return np.maximum(np.ldexp(1.0, e - 8), 2.0 ** -133)


def _sum_error_bound(x, w, shape):
    """hidden * 2^-23 * sum_c |x[b, c]| |w[n, c]|, shaped like the projection."""
    ax, aw = np.abs(to_f64(x)), np.abs(to_f64(w))
    return (x.shape[1] * 2.0 ** -23 * (ax @ aw.T)).reshape(shape)


def assert_projection(gpu, ref, what, x, w):
    g = gpu.double().cpu().numpy()
    assert np.isfinite(g).all(), f"{what}: non-finite projection"
    diff = np.abs(g - ref)
    bound = _bf16_spacing(np.maximum(np.abs(g), np.abs(ref))) + _sum_error_bound(x, w, g.shape)
    assert (diff <= bound).all(), f"{what}: max |gpu-ref| / bound = {np.max(diff / bound):.2f}"
    exact = float(np.mean(diff == 0))
    assert exact >= 0.99, f"{what}: only {exact:.4f} of the elements equal the oracle's rounding"


def _all_heads(B, Hq):
    return [(b, h) for b in range(B) for h in range(Hq)]


# ----------------------------------------------------------------- workload

def test_decode_projected_workload(px):
    w = W.WORKLOADS["decode_projected"]
    inp = W.projected_decode_inputs(w, device=DEV)
    out, q, rho = _run(px, inp)
    qr, rr, ref = _oracle(inp)
    assert_projection(q, qr, "q", inp["x"], inp["w_q"])
    assert_projection(rho, rr, "rho", inp["x"], inp["w_rho"])
    assert out.dtype == torch.bfloat16
    assert_parity(out.float().cpu().numpy(), ref, TOL_BF16, "decode_projected")
    assert px.last_device_error() == 0


# ------------------------------------------------------------------- sweeps

@pytest.mark.parametrize("B,Hq,Hkv,d,L,hidden", [
    (1, 2, 1, 64, 65, 32),          # one 32-column chunk
    (3, 4, 2, 128, 200, 96),        # fewer chunks than warps
    (9, 8, 2, 64, 1000, 256),       # ragged second batch tile
    (17, 4, 4, 128, 130, 544),      # partial unrolled group of chunks
    (40, 2, 1, 64, 64, 2048),
    (70, 4, 2, 128, 300, 160),      # batch rows past one CTA's 64: two grid rows
])
def test_shapes(px, B, Hq, Hkv, d, L, hidden):
    inp = _inputs(B, Hq, Hkv, d, L, hidden, seed=B * 1000 + hidden)
    out, q, rho = _run(px, inp, out_dtype=torch.float32)
    qr, rr, ref = _oracle(inp)
    assert_projection(q, qr, "q", inp["x"], inp["w_q"])
    assert_projection(rho, rr, "rho", inp["x"], inp["w_rho"])
    assert_parity(out.cpu().numpy(), ref, TOL_BF16, f"B={B} Hq={Hq} d={d} L={L} hidden={hidden}")


def test_paged_ragged_with_empty_sequences(px):
    lens = [0, 1, 130, 64, 0, 257]
    inp = _inputs(6, 8, 2, 128, 300, 512, seed=77, seq_lens=lens, paged=True)
    out, q, rho = _run(px, inp, out_dtype=torch.float32)
    qr, rr, ref = _oracle(inp)
    assert_projection(q, qr, "q", inp["x"], inp["w_q"])
    assert_projection(rho, rr, "rho", inp["x"], inp["w_rho"])
    o = out.cpu().numpy()
    assert not o[0].any() and not o[4].any()
    assert_parity(o, ref, TOL_BF16, "paged ragged")
    assert px.last_device_error() == 0


def test_zero_probe_weights(px):
    inp = _inputs(4, 8, 4, 128, 500, 256, seed=5)
    inp["w_rho"] = torch.zeros_like(inp["w_rho"])
    out, q, rho = _run(px, inp, out_dtype=torch.float32)
    assert not rho.any()
    _, _, ref = _oracle(inp)
    assert_parity(out.cpu().numpy(), ref, TOL_BF16, "rho = 0")


# ------------------------------------------------------- launch dependency

def test_matches_plain_decode_of_its_projections_with_stale_buffers(px):
    inp = _inputs(8, 16, 8, 128, 4096, 2048, seed=11)
    q_out = torch.full((8, 16, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
    rho_out = torch.full_like(q_out, float("nan"))
    out, q, rho = _run(px, inp, q_out=q_out, rho_out=rho_out)
    torch.cuda.synchronize()
    assert torch.isfinite(out.float()).all()
    plain = px.decode(q.clone(), rho.clone(), inp["k_cache"], inp["v_cache"], inp["scale"])
    assert torch.equal(out, plain)


def test_back_to_back_calls_on_shared_buffers(px):
    base = _inputs(8, 16, 8, 128, 1024, 2048, seed=21)
    xs = [W.projection_inputs(8, 16, 128, 2048, device=DEV, seed=100 + i)["x"] for i in range(6)]
    q_out = torch.empty((8, 16, 128), dtype=torch.bfloat16, device=DEV)
    rho_out = torch.empty_like(q_out)
    outs = []
    for x in xs:   # no synchronisation between calls; q_out / rho_out reused
        o, _, _ = px.decode_projected(x, base["w_q"], base["w_rho"], base["k_cache"], base["v_cache"],
                                      base["scale"], q_out=q_out, rho_out=rho_out)
        outs.append(o)
    torch.cuda.synchronize()
    for x, o in zip(xs, outs):
        want, q, rho = px.decode_projected(x, base["w_q"], base["w_rho"], base["k_cache"], base["v_cache"],
                                           base["scale"])
        torch.cuda.synchronize()
        assert torch.equal(o, want)
    assert px.last_device_error() == 0


def test_graph_replay_with_new_inputs(px):
    inp = _inputs(8, 16, 8, 128, 2048, 2048, seed=31)
    x_static = inp["x"].clone()
    q_out = torch.empty((8, 16, 128), dtype=torch.bfloat16, device=DEV)
    rho_out = torch.empty_like(q_out)
    out = torch.empty_like(q_out)

    def call():
        px.decode_projected(x_static, inp["w_q"], inp["w_rho"], inp["k_cache"], inp["v_cache"], inp["scale"],
                            q_out=q_out, rho_out=rho_out, out=out)

    call()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    for i in range(3):
        x = W.projection_inputs(8, 16, 128, 2048, device=DEV, seed=200 + i)["x"]
        x_static.copy_(x)
        q_out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        case = dict(inp, x=x)
        qr, rr, ref = _oracle(case, heads=[(0, 0), (3, 7), (7, 15)])
        assert_projection(q_out, qr, f"graph q {i}", x, inp["w_q"])
        assert_projection(rho_out, rr, f"graph rho {i}", x, inp["w_rho"])
        o = out.float().cpu().numpy()
        for b, h in [(0, 0), (3, 7), (7, 15)]:
            assert_parity(o[b, h], ref[b, h], TOL_BF16, f"graph replay {i} ({b},{h})")
    assert px.last_device_error() == 0
