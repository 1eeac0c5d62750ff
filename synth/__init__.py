"""Seeded synthetic inputs shared by the CPU oracle's tests and the CUDA path.

This package draws random numbers, mixes them through seeded low-rank factors, rounds them to
bf16 once and lays them out in a paged cache. It holds none of the sparse-attention method's own
arithmetic (no projection, scoring, selection or attention), so both sides can use it without
sharing any step of the computation under test.
"""

from .generator import (  # noqa: F401
    WORKLOADS,
    Workload,
    layer_factors,
    sample_calibration,
    sample_decode_queries,
    build_paged_kv,
    page_permutation,
    torch_generator,
)
