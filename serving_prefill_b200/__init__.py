"""Precomputed-KV RAG prefill on B200 (sm_100a).

The hot path (paged gather, causal attention over the concatenated chunk
caches, CacheBlend Impact, top-k recompute selection) runs in the CUDA
kernels of librag.so behind the C ABI of include/rag_prefill.h; this package
is its thin ctypes binding.
"""

from .rag import (  # noqa: F401
    Batch,
    KVPool,
    RagError,
    lib,
    new_workspace,
    rag_abi_version,
    rag_fused_prefill_attn,
    rag_fused_prefill_attn_rope,
    rag_impact_topk,
    rag_kv_decode,
    rag_kv_pool_write,
    rag_last_device_error,
    rag_launch_count,
    rag_num_sms,
    rag_profile_collect,
    rag_profile_peek,
    rag_profile_enable,
    rag_recompute_count,
    rag_recompute_kv,
    rag_recompute_plan,
    rag_recompute_plan_size,
    rag_recompute_status,
    rag_workspace_size,
    topk_capacity,
)
