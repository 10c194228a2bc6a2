"""Seeded synthetic inputs for precomputed-KV RAG prefill.

This package draws random numbers and lays out the inputs (chunk lengths,
physical page assignment, batch descriptors, per-layer K/V/Q values). It holds
none of the method's arithmetic: the CUDA path and the CPU oracle both consume
what it produces, and neither is imported from here.
"""

from .rag import (  # noqa: F401
    PAGE_SIZE,
    WORKLOADS,
    Workload,
    BatchLayout,
    LayerInputs,
    RecomputeInputs,
    make_recompute_inputs,
    random_selection,
    make_encoded_layer,
    make_layout,
    make_layer_inputs,
    get_workload,
    scaled,
)
