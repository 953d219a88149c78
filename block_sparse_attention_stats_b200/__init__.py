"""PISA piecewise sparse attention on NVIDIA B200 (sm_100a).

The compute lives in libpisa.so (hand-written CUDA kernels behind the C ABI of
include/pisa.h); this package is its thin Python binding.
"""
from .api import (  # noqa: F401
    PisaError,
    piecewise_sparse_attention,
    piecewise_sparse_attention_0th,
    piecewise_sparse_attention_hyd,
    pisa_attention,
    pisa_attention_ex,
    pisa_block_stats,
    pisa_block_stats_noalloc,
    pisa_dense_attention,
    pisa_device_status,
    pisa_num_blocks,
    pisa_num_selected,
    pisa_select,
    pisa_selftest_timeout,
    pisa_sparse_attention,
    pisa_sparse_attention_bwd,
    pisa_sparse_attention_fwd,
    pisa_tail_score_histogram,
    pisa_workspace_bytes,
)
