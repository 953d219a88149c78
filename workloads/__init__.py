"""Seeded synthetic workloads for PISA piecewise sparse attention.

This package holds the input generator shared by the oracle-based tests and the
GPU path (tests, ``bench.py``). It contains none of the attention method's
arithmetic: only random numbers, cluster layouts and the workload shapes.
"""
from .generator import (  # noqa: F401
    WORKLOADS,
    Workload,
    cluster_map,
    generate_head,
    generate_qkv,
    stream_normal,
    stream_uniform_u64,
)
