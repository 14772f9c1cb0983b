"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the CPU oracle.

This package draws random numbers and lays them out; it holds none of the
method's arithmetic (no prediction, scoring, selection or attention).
"""
from .workloads import (  # noqa: F401
    WORKLOADS,
    Workload,
    workload,
    kv_cache,
    query_history,
    score_rows,
    random_selection,
)
