"""Device-resident state for one batch and the whole prefill step.

`PrefillEngine` owns the caller-side buffers of the C ABI (workspace, outputs)
for a pool and a batch, and runs a step: the fused attention of every layer,
Impact on the selecting layer, then the top-k recompute selection. Each call
is one or more librag.so launches on the current stream.
"""

from __future__ import annotations

import torch

from .rag import (Batch, KVPool, new_workspace, rag_fused_prefill_attn, rag_impact_topk, rag_kv_pool_write,
                  rag_last_device_error, topk_capacity)


def write_chunks(pool: KVPool, layer: int, chunk_pages, chunk_k, chunk_v, device_err=None):
    """Store every chunk's dense K/V of one layer into its pages."""
    for pages, k, v in zip(chunk_pages, chunk_k, chunk_v):
        rag_kv_pool_write(pool, layer, pages, k, v, device_err=device_err)


class PrefillEngine:
    def __init__(self, pool: KVPool, batch: Batch, num_q_heads: int, r: float, dtype=torch.bfloat16,
                 device="cuda"):
        self.pool, self.batch, self.r = pool, batch, r
        hd = pool.c.head_dim
        self.num_q_heads = num_q_heads
        self.ws = new_workspace(pool, batch, num_q_heads, device=device)
        tq = batch.total_q
        self.o = torch.empty(max(tq, 1), num_q_heads, hd, dtype=dtype, device=device)
        self.row_lse = torch.empty(max(tq, 1), num_q_heads, dtype=torch.float32, device=device)
        self.impact = torch.empty(max(batch.total_doc + tq, 1), dtype=torch.float32, device=device)
        self.k_cap = topk_capacity(batch, r)
        B = max(batch.num_requests, 1)
        self.topk_idx = torch.empty(B, self.k_cap, dtype=torch.int32, device=device)
        self.topk_val = torch.empty(B, self.k_cap, dtype=torch.float32, device=device)
        self.k = torch.empty(B, dtype=torch.int32, device=device)

    def attend(self, layer: int, q, kq, vq, with_impact: bool, o=None, row_lse=None):
        rag_fused_prefill_attn(self.pool, layer, self.batch, q, kq, vq, self.o if o is None else o, self.ws,
                               impact=self.impact if with_impact else None,
                               row_lse=self.row_lse if row_lse is None else row_lse)

    def select(self):
        rag_impact_topk(self.impact, self.batch, self.r, self.k_cap, self.topk_idx, self.topk_val, self.k)

    def step(self, layers, impact_layer, outs=None):
        """layers: list of (layer index, q, kq, vq). outs: optional per-layer O buffers.
        impact_layer: the layer that feeds Impact and the top-k, or None (decode:
        attention only)."""
        for n, (layer, q, kq, vq) in enumerate(layers):
            self.attend(layer, q, kq, vq, with_impact=(layer == impact_layer),
                        o=None if outs is None else outs[n])
        if impact_layer is not None:
            self.select()

    def device_error(self):
        return rag_last_device_error(self.ws)
