"""DashAttention forward oracle: TEST INFRASTRUCTURE ONLY.

A plain, slow, fp64 CPU restatement of what the DashAttention forward path
computes (chunk summary, alpha-entmax routing with GQA averaging, and the
prior-induced block-sparse softmax), written from the text of the pages on
"DashAttention: Differentiable and Adaptive Sparse Hierarchical Attention".

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the C-ABI library and
its Python binding) never imports it and has no CPU fallback.

Pins (checked by ``tests/test_oracle.py`` against something other than the
oracle itself): see the module docstring of :mod:`oracle.dash_oracle`.  The
gradients of the path (:mod:`oracle.dash_oracle_bwd`) are pinned by finite
differences of the forward functions in ``tests/test_oracle_bwd.py``.

parity unpinned: the authors' exact form of the prior g, of the strength sigma
and of the diagonal branch.  The pages leave these open; the oracle fixes one
documented reading (g uniform within a block and proportional to w_b**sigma,
diagonal block always on with weight 1) and only that reading is pinned.
"""

from .dash_oracle import (  # noqa: F401
    entmax_bisect,
    entmax15_sort,
    chunk_summary,
    diagonal_summary,
    summarize_append,
    route,
    route_topk,
    pack_mask,
    pack_weights,
    unpack_weights,
    unpack_mask,
    attn_fwd,
    decode,
    decode_varlen,
    decode_paged,
    decode_attend,
    gather_pages,
)
