"""Shared test helpers: float64 views of device tensors and the parity check."""

import numpy as np
import torch

# Tolerances fixed by the method's accuracy target: max |gpu - ref| <= tol * (1 + |ref|)
TOL_F32 = 1e-5
TOL_BF16 = 2e-2


class F64View:
    """Read-only float64 numpy view of a (possibly device-resident) tensor.

    Indexing copies just the selected slice to the host, so the oracle can
    walk a multi-GiB cache one sequence or page at a time.
    """

    def __init__(self, t):
        self.t = t
        self.shape = tuple(t.shape)

    def __getitem__(self, idx):
        return self.t[idx].double().cpu().numpy()


def to_f64(t):
    return t.double().cpu().numpy()


def parity_error(gpu, ref):
    """max over elements of |gpu - ref| / (1 + |ref|); NaN anywhere gives inf."""
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    if not np.isfinite(g).all() or not np.isfinite(r).all():
        return float("inf")
    return float(np.max(np.abs(g - r) / (1.0 + np.abs(r)))) if g.size else 0.0


def assert_parity(gpu, ref, tol, what=""):
    err = parity_error(gpu, ref)
    assert err <= tol, f"{what}: max |gpu-ref|/(1+|ref|) = {err:.3e} > {tol:.1e}"
    return err


def oracle_heads(inp, heads):
    """Oracle decode of selected (b, h) for an input dict from workloads."""
    import oracle
    q = to_f64(inp["q"])
    rho = to_f64(inp["rho"])
    lens = None if inp.get("seq_lens") is None else inp["seq_lens"].cpu().numpy()
    table = None if inp.get("page_table") is None else inp["page_table"].cpu().numpy()
    return oracle.decode(q, rho, F64View(inp["k_cache"]), F64View(inp["v_cache"]), inp["scale"],
                         seq_lens=lens, page_table=table, heads=heads)
