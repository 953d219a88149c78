"""fp64 CPU oracle of PISA piecewise sparse attention.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
product (the CUDA library and its Python binding) never calls it, and it shares
no code with the CUDA path.
"""
from .pisa_oracle import (  # noqa: F401
    block_partition,
    block_stats,
    covariance_norms,
    dense_attention,
    num_selected,
    piecewise_attention,
    pisa_attention_head,
    pisa_attention,
    selection_scores,
    select_blocks,
    tail_score_histogram,
)
from .pisa_backward import zeroth_order_backward, zeroth_order_forward  # noqa: F401
