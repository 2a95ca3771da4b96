"""GPU parity of the prefill backward (and the training forward) against the
float64 oracle.

Gradients of sum(dout * out) from parallax_prefill_train +
parallax_prefill_backward are compared with torch float64 autograd through
the explicit definition (oracle.prefill_grads), on the same seeded bf16
inputs:  max |gpu - ref| <= 2e-2 * (1 + |ref|)  (bf16 operands, fp32
accumulation), for dq, drho, dk and dv.  Lengths cover one row, partial and
full 64/128 tiles and ragged tails; grouped KV heads, full attention and
unit-scale probes are covered; the full B=4, H=16, T=8192 workload is
checked on sampled rows (dq, drho) and keys (dk, dv).
"""

import numpy as np
import pytest
import torch

import oracle
from parallax_local_linear_b200 import workloads as W
from tests.helpers import TOL_BF16, F64View, assert_parity, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def px():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from parallax_local_linear_b200 import binding
    return binding


def _inputs(B, H, T, Hkv=0, seed=0, rho_scale=0.1):
    x = W.small_prefill_inputs(B, H, T, 128, num_kv_heads=Hkv, rho_scale=rho_scale, seed=seed)
    x = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    x["dout"] = W.dout_like(x["q"], seed + 1000)
    return x


def _gpu_grads(px, x, causal=True):
    out, vbar, stats = px.prefill_train(x["q"], x["rho"], x["k"], x["v"], causal, x["scale"], out_dtype=torch.float32)
    return px.prefill_backward(x["q"], x["rho"], x["k"], x["v"], out, vbar, stats, x["dout"], causal, x["scale"])


def _check(px, x, causal=True, what=""):
    grads = _gpu_grads(px, x, causal)
    ref = oracle.prefill_grads(*(to_f64(x[k]) for k in ("q", "rho", "k", "v", "dout")), x["scale"], causal=causal)
    for name, gg, rr in zip(("dq", "drho", "dk", "dv"), grads, ref):
        assert_parity(gg.cpu().numpy(), rr, TOL_BF16, f"{name} {what}")
    assert px.last_device_error() == 0


@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 127, 128, 129, 200])
def test_causal_grads(px, T):
    _check(px, _inputs(1, 2, T, seed=T), what=f"T={T}")


def test_batch_and_full_attention(px):
    _check(px, _inputs(2, 2, 70, seed=3), what="B=2")
    _check(px, _inputs(1, 2, 100, seed=4), causal=False, what="non-causal")


def test_grouped_kv_heads(px):
    _check(px, _inputs(1, 4, 130, Hkv=2, seed=5), what="gqa")


def test_unit_scale_probe(px):
    _check(px, _inputs(1, 2, 150, seed=6, rho_scale=1.0), what="unit rho")


@pytest.mark.parametrize("pair", [False, True])
def test_training_forward_outputs(px, pair):
    x = _inputs(1, 2, 300, seed=7)
    out, vbar, stats = px.prefill_train(x["q"], x["rho"], x["k"], x["v"], True, x["scale"], out_dtype=torch.float32,
                                        cta_pair=pair)
    plain = px.prefill(x["q"], x["rho"], x["k"], x["v"], causal=True, scale=x["scale"], out_dtype=torch.float32,
                       cta_pair=pair)
    assert torch.equal(out, plain)
    q, rho, k, v = (to_f64(x[n]) for n in ("q", "rho", "k", "v"))
    st = stats.cpu().numpy().astype(np.float64)
    vb = vbar.cpu().numpy().astype(np.float64)
    for h in range(2):
        for t in (0, 1, 63, 64, 150, 299):
            s = x["scale"] * k[0, h, :t + 1] @ q[0, h, t]
            w = oracle.softmax_weights(s)
            np.testing.assert_allclose(vb[0, h, t], w @ v[0, h, :t + 1], rtol=0, atol=2e-2)
            np.testing.assert_allclose(st[0, h, t, 1], w @ (k[0, h, :t + 1] @ rho[0, h, t]), rtol=0, atol=2e-2)
            # the weights 2^(scale log2(e) q.k - x) sum to one
            total = np.sum(np.exp2(s * np.log2(np.e) - st[0, h, t, 0]))
            assert abs(total - 1.0) < 1e-3, (h, t, total)


def test_autograd_function(px):
    x = _inputs(1, 2, 90, seed=8)
    leaves = [x[n].clone().requires_grad_(True) for n in ("q", "rho", "k", "v")]
    out = px.ParallaxPrefill.apply(*leaves, True, x["scale"])
    out.backward(x["dout"])
    o2, vb, st = px.prefill_train(x["q"], x["rho"], x["k"], x["v"], True, x["scale"])
    ref = px.prefill_backward(x["q"], x["rho"], x["k"], x["v"], o2, vb, st, x["dout"], True, x["scale"])
    for leaf, r in zip(leaves, ref):
        assert leaf.grad.dtype == torch.bfloat16
        assert torch.equal(leaf.grad, r)


def test_deterministic(px):
    x = _inputs(1, 2, 257, seed=9)
    a = _gpu_grads(px, x)
    b = _gpu_grads(px, x)
    for ga, gb in zip(a, b):
        assert torch.equal(ga, gb)


def test_full_prefill_workload_sampled(px):
    from tests.test_prefill_gpu import full_workload_rows
    w = W.WORKLOADS["prefill"]
    x = W.prefill_inputs(w, device="cuda")
    dout = W.dout_like(x["q"], w.seed + 1000)
    out, vbar, stats = px.prefill_train(x["q"], x["rho"], x["k"], x["v"], True, x["scale"])
    dq, drho, dk, dv = px.prefill_backward(x["q"], x["rho"], x["k"], x["v"], out, vbar, stats, dout, True,
                                           x["scale"])
    for gg in (dq, drho, dk, dv):
        assert torch.isfinite(gg.float()).all()
    T, tail = w.seq_len, 65
    rows = full_workload_rows(w.batch, w.num_heads, T)
    pairs = sorted({(b, h) for b, h, _ in rows})
    for n_pair, (b, h) in enumerate(pairs):
        sl = {k: x[k][b, h].double().cpu().numpy() for k in ("q", "rho", "k", "v")}
        g = dout[b, h].double().cpu().numpy()
        ts = sorted({t for bb, hh, t in rows if (bb, hh) == (b, h)})
        # in half of the pairs the last `tail` rows are all computed: they give
        # dk, dv of the last `tail` keys exactly (no earlier row sees them)
        full_tail = n_pair % 2 == 0
        if full_tail:
            ts = sorted(set(ts) | set(range(T - tail, T)))
        sk = np.zeros((tail, 128))
        sv = np.zeros((tail, 128))
        rq_all, rr_all = {}, {}
        for t in ts:
            rq, rr, rk, rv = oracle.query_grads(sl["q"][t], sl["rho"][t], sl["k"][:t + 1], sl["v"][:t + 1], g[t],
                                                x["scale"])
            rq_all[t], rr_all[t] = rq, rr
            if full_tail and t >= T - tail:
                sk[: t + 1 - (T - tail)] += rk[T - tail:]
                sv[: t + 1 - (T - tail)] += rv[T - tail:]
        got_q = dq[b, h, ts].float().cpu().numpy()
        got_r = drho[b, h, ts].float().cpu().numpy()
        assert_parity(got_q, np.stack([rq_all[t] for t in ts]), TOL_BF16, f"dq (b={b}, h={h})")
        assert_parity(got_r, np.stack([rr_all[t] for t in ts]), TOL_BF16, f"drho (b={b}, h={h})")
        if full_tail:
            assert_parity(dk[b, h, T - tail:].float().cpu().numpy(), sk, TOL_BF16, f"dk (b={b}, h={h})")
            assert_parity(dv[b, h, T - tail:].float().cpu().numpy(), sv, TOL_BF16, f"dv (b={b}, h={h})")
    assert px.last_device_error() == 0
