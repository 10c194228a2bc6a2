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


class HostStep:
    """A whole step from pinned host buffers to pinned host buffers.

    The batch descriptors and every layer's q, kq, vq travel host -> device on
    a copy stream, each layer's O travels back on a second one, and the
    kernels run on the caller's current stream; events order them, so layer
    l + 1's inputs arrive, and layer l - 1's output leaves, while layer l
    computes (and the next step's copies start as soon as the buffers they
    overwrite are free). Every step of the method still runs in the library's
    kernels; this class only schedules the copies around them.
    """

    def __init__(self, engine: "PrefillEngine", layers_dev, outs_dev, host_in, host_out, impact_layer,
                 host_topk=None, batch_host=None):
        self.eng = engine
        self.layers_dev = layers_dev        # [(layer, q, kq, vq)] device buffers
        self.outs_dev = outs_dev            # per layer device O
        self.host_in = host_in              # per layer (q, kq, vq) pinned host tensors
        self.host_out = host_out            # per layer pinned host O
        self.impact_layer = impact_layer
        self.host_topk = host_topk
        self.batch_host = batch_host        # pinned host copies of the batch descriptor arrays, or None
        self.s_in = torch.cuda.Stream()
        self.s_out = torch.cuda.Stream()
        n = len(layers_dev)
        self.ev_in = [torch.cuda.Event() for _ in range(n)]
        self.ev_done = [torch.cuda.Event() for _ in range(n)]
        self.ev_out = [torch.cuda.Event() for _ in range(n)]
        self.ev_desc = torch.cuda.Event()
        self.ev_step = torch.cuda.Event()
        self.started = False

    def __call__(self):
        cur = torch.cuda.current_stream()
        n = len(self.layers_dev)
        with torch.cuda.stream(self.s_in):
            # a step's copies begin after everything the caller queued before it
            self.s_in.wait_stream(cur)
            if self.batch_host is not None:
                if self.started:
                    self.s_in.wait_event(self.ev_step)     # the previous step no longer reads them
                for t, dt in zip(self.batch_host, self.eng.batch.dev):
                    if t.numel():
                        dt[: t.numel()].copy_(t, non_blocking=True)
                self.ev_desc.record(self.s_in)
            for i in range(n):
                if self.started:
                    self.s_in.wait_event(self.ev_done[i])  # the previous step's layer i has read them
                _, q, kq, vq = self.layers_dev[i]
                hq, hkq, hvq = self.host_in[i]
                q.copy_(hq, non_blocking=True)
                kq.copy_(hkq, non_blocking=True)
                vq.copy_(hvq, non_blocking=True)
                self.ev_in[i].record(self.s_in)
        if self.batch_host is not None:
            cur.wait_event(self.ev_desc)
        for i in range(n):
            layer, q, kq, vq = self.layers_dev[i]
            cur.wait_event(self.ev_in[i])
            if self.started:
                cur.wait_event(self.ev_out[i])             # the previous step's O of this layer has left
            self.eng.attend(layer, q, kq, vq, with_impact=(layer == self.impact_layer), o=self.outs_dev[i])
            self.ev_done[i].record(cur)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(self.ev_done[i])
                self.host_out[i].copy_(self.outs_dev[i], non_blocking=True)
                self.ev_out[i].record(self.s_out)
        if self.impact_layer is not None:
            self.eng.select()
            if self.host_topk is not None:
                self.host_topk.copy_(self.eng.topk_idx, non_blocking=True)
        self.ev_step.record(cur)
        cur.wait_stream(self.s_out)                        # the step ends when its last output has left
        self.started = True
