"""Seeded synthetic inputs shared by the oracle tests, the CUDA parity tests and the benchmark.

This package draws random numbers and lays them out; it holds none of the codec's arithmetic
(no decomposition, rotation, quantisation, allocation or attention).
"""
from .workloads import WORKLOADS, Workload, get_workload  # noqa: F401
from .gen import (  # noqa: F401
    make_kv,
    make_kv_cell,
    make_queries,
    make_inv_freq,
    make_gaussian_rows,
    make_random_tables,
    make_random_cache_parts,
)
