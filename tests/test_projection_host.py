"""Host-side checks of the projected decode that need no GPU: the seeded
inputs, the algorithmic byte count, the binding's argument checks, and the
oracle leg of bench.py on a small projected workload."""

import dataclasses

import numpy as np
import pytest
import torch

from parallax_local_linear_b200 import workloads as W


def test_projection_inputs_are_seeded_bf16_with_unit_variance_outputs():
    a = W.projection_inputs(4, 8, 64, 512, seed=3)
    b = W.projection_inputs(4, 8, 64, 512, seed=3)
    c = W.projection_inputs(4, 8, 64, 512, seed=4)
    assert a["x"].shape == (4, 512) and a["w_q"].shape == (512, 512) and a["w_rho"].shape == (512, 512)
    assert all(t.dtype == torch.bfloat16 for t in a.values())
    assert all(torch.equal(a[k], b[k]) for k in a)
    assert not torch.equal(a["x"], c["x"])
    assert not torch.equal(a["w_q"], a["w_rho"])
    # W ~ N(0, 1/hidden): every projected component has variance ~1
    q = a["x"].double() @ a["w_q"].double().T
    assert 0.8 < float(q.var()) < 1.25


def test_projected_workload_inputs_extend_the_decode_inputs():
    w = W.WORKLOADS["decode_projected"]
    small = dataclasses.replace(w, batch=2, kv_len=128)
    inp = W.projected_decode_inputs(small)
    plain = W.decode_inputs(small)
    assert torch.equal(inp["k_cache"], plain["k_cache"]) and torch.equal(inp["v_cache"], plain["v_cache"])
    assert inp["x"].shape == (2, w.hidden)
    assert inp["w_q"].shape == (w.num_q_heads * w.head_dim, w.hidden)


def test_projection_bytes():
    # two [n, hidden] bf16 weights and x read, q and rho written
    B, Hq, d, hidden = 8, 16, 128, 2048
    n = Hq * d
    assert W.projection_bytes(B, Hq, d, hidden) == 2 * (2 * n * hidden + B * hidden + 2 * B * n)
    assert W.projection_bytes(B, Hq, d, hidden) == 16_875_520


def test_binding_rejects_host_tensors_before_calling_the_library():
    from parallax_local_linear_b200 import binding as px
    inp = W.small_decode_inputs(1, 2, 1, 64, 64, seed=0)
    pj = W.projection_inputs(1, 2, 64, 64, seed=1)
    with pytest.raises(ValueError, match="CUDA"):
        px.decode_projected(pj["x"], pj["w_q"], pj["w_rho"], inp["k_cache"], inp["v_cache"])


def test_oracle_leg_counts_the_projection_once_per_step():
    import bench
    w = dataclasses.replace(W.WORKLOADS["decode_projected"], batch=2, num_q_heads=4, num_kv_heads=2,
                            head_dim=64, kv_len=128, hidden=64)
    inp = W.projected_decode_inputs(w)
    gbs, secs, done, desc = bench.oracle_decode_sample(w, inp, budget_s=60.0)
    assert done == w.batch * w.num_kv_heads
    want = (W.kv_bytes(w) + W.projection_bytes(w.batch, w.num_q_heads, w.head_dim, w.hidden)) / secs / 1e9
    assert np.isclose(gbs, want, rtol=1e-9)
    assert "projection" in desc


# --------------------------------------------------------------------------
# Binding checks of caller buffers (host logic; the CUDA check comes last)
# --------------------------------------------------------------------------

def test_output_buffer_shape_and_dtype_are_checked_before_any_launch():
    from parallax_local_linear_b200 import binding as px
    with pytest.raises(ValueError, match="shape"):
        px._output(torch.empty(2, 3, 4), None, (2, 3, 5), torch.bfloat16, "cpu")
    with pytest.raises(TypeError, match="out_dtype"):
        px._output(torch.empty(2, 3, 4), torch.bfloat16, (2, 3, 4), torch.bfloat16, "cpu")
    with pytest.raises(ValueError, match="CUDA"):   # right shape and dtype: only the device is wrong
        px._output(torch.empty(2, 3, 4), None, (2, 3, 4), torch.bfloat16, "cpu")
    out, dt = px._output(None, None, (2, 3), torch.float32, "cpu")
    assert out.shape == (2, 3) and dt == torch.float32


def test_sequence_tables_are_checked_against_the_batch():
    from parallax_local_linear_b200 import binding as px
    lens = torch.zeros(3, dtype=torch.int32)
    table = torch.zeros(3, 5, dtype=torch.int32)
    with pytest.raises(ValueError, match="seq_lens must have shape"):
        px._check_sequences(4, lens, None)
    with pytest.raises(ValueError, match="page_table must be"):
        px._check_sequences(4, torch.zeros(4, dtype=torch.int32), table)
    with pytest.raises(ValueError, match="needs seq_lens"):
        px._check_sequences(3, None, table)
    with pytest.raises(ValueError, match="CUDA"):
        px._check_sequences(3, lens, table)
