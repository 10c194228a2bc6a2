"""CPU fp64 oracle for precomputed-KV RAG prefill — TEST INFRASTRUCTURE ONLY.

This package is the plain, slow definition that the CUDA path is checked
against. Only `tests/`, the smoke check and the benchmark's CPU-baseline leg
may import it; the library path never does and has no CPU fallback.
"""

from .prefill import (  # noqa: F401
    pool_write,
    gather,
    recompute_count,
    attend_request,
    select_topk,
    run_workload_layer,
    run_workload,
    OracleResult,
)
from . import recompute  # noqa: F401
