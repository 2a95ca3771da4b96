"""Float64 CPU oracle for Parallax attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` use it.  It shares no code with
the CUDA library (no kernels, headers, helpers or constants) and imports
nothing from ``parallax_local_linear_b200``.

Sources (web pages on the method):
  * "Parallax: Parameterized Local Linear Attention for Language Modeling"
    (newx.sg paper page), section "Abstract".
  * "Parallax: Breaking the Boundary Bias with Parameterized Local Linear
    Attention" (wispaper.ai blog), sections "Context: Why Softmax is Not
    Enough", "The Core Insight: Covariance Correction" and "Hardware
    Efficiency".
  * Local Linear Attention with the solved probe (``lla_*``): the newx.sg
    "Abstract" and the blog's "Context" section.
"""

from .parallax_oracle import (  # noqa: F401
    softmax_weights,
    parallax_query,
    sigma_kv,
    decode,
    gather_paged_keys,
    prefill_rows,
    prefill_paged_rows,
    prefill_grads,
    query_grads,
    round_bf16,
    project_heads,
    decode_projected,
    sigma_kk,
    lla_probe,
    lla_query,
    lla_decode,
)
