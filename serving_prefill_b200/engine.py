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


def layer_groups(per_layer, group_size, device, fill=True):
    """Pack per-layer tensors into one pinned host buffer and one device buffer
    per group of `group_size` consecutive layers (the layout HostStep copies
    in one piece). per_layer[i] is a tuple of tensors of layer i (host or
    device, any dtype); each gets a 256-byte aligned slot. Returns
    (groups, host_views, dev_views): groups as HostStep's in_groups /
    out_groups take them (host buffer, device buffer, [layer positions]), and
    per layer the tuples of host and device views. fill copies the tensors'
    values into the host views."""
    groups, host_views, dev_views = [], [], []
    for g0 in range(0, len(per_layer), group_size):
        idx = list(range(g0, min(g0 + group_size, len(per_layer))))
        offs, at = [], 0
        for i in idx:
            row = []
            for t in per_layer[i]:
                row.append(at)
                at += (t.numel() * t.element_size() + 255) // 256 * 256
            offs.append(row)
        host = torch.empty(max(at, 256), dtype=torch.uint8).pin_memory()
        dev = torch.empty(max(at, 256), dtype=torch.uint8, device=device)
        for i, row in zip(idx, offs):
            hv, dv = [], []
            for t, o in zip(per_layer[i], row):
                nb = t.numel() * t.element_size()
                h = host[o:o + nb].view(t.dtype).view(t.shape)
                if fill:
                    h.copy_(t)
                hv.append(h)
                dv.append(dev[o:o + nb].view(t.dtype).view(t.shape))
            host_views.append(tuple(hv))
            dev_views.append(tuple(dv))
        groups.append((host, dev, idx))
    return groups, host_views, dev_views


class HostStep:
    """A whole step from pinned host buffers to pinned host buffers.

    The batch descriptors and every layer's q, kq, vq travel host -> device on
    copy streams, each layer's O travels back on another one, and the kernels
    run on the caller's current stream; events order them, so later layers'
    inputs arrive, and earlier layers' outputs leave, while a layer computes.
    Every step of the method still runs in the library's kernels; this class
    only schedules the copies around them. A step's host outputs are complete
    once host_ready() (an event on the output copy stream) has completed.

    Copies go either per tensor (host_in[i] = (q, kq, vq), host_out[i]) or, with
    in_groups / out_groups, per group of consecutive layers: a group is
    (host buffer, device buffer, [layer positions]) whose layers' device q, kq,
    vq (or O) are views of the device buffer laid out like the host buffer, so
    the group moves in one copy and the kernels of its layers follow one
    another with no event wait between them.

    depth = 2 keeps a second set of device inputs, outputs and batch
    descriptors, and consecutive steps alternate between the two sets: a
    step's uploads then wait only for the step before the previous one, so
    they run while the previous step computes. The host buffers are shared by
    both sets: a caller that rewrites them between steps waits for the copies
    of the step that read them (host_ready() of that step covers them).
    """

    def __init__(self, engine: "PrefillEngine", layers_dev, outs_dev, host_in, host_out, impact_layer,
                 host_topk=None, batch_host=None, in_groups=None, out_groups=None, depth=1):
        assert depth in (1, 2)
        self.eng = engine
        self.impact_layer = impact_layer
        self.host_topk = host_topk
        self.batch_host = batch_host        # pinned host copies of the batch descriptor arrays, or None
        n = len(layers_dev)
        if in_groups is None:
            in_groups = [(host_in[i], layers_dev[i][1:], [i]) for i in range(n)]
        if out_groups is None:
            out_groups = [(host_out[i], outs_dev[i], [i]) for i in range(n)]
        for groups in (in_groups, out_groups):
            order = [i for _, _, idx in groups for i in idx]
            assert order == list(range(n)), "groups must cover the layers in order"
        self.in_first = {idx[0]: g for g, (_, _, idx) in enumerate(in_groups)}
        self.in_last = {idx[-1]: g for g, (_, _, idx) in enumerate(in_groups)}
        self.out_first = {idx[0]: g for g, (_, _, idx) in enumerate(out_groups)}
        self.out_last = {idx[-1]: g for g, (_, _, idx) in enumerate(out_groups)}
        self.sets = [self._new_set(layers_dev, outs_dev, in_groups, out_groups, engine.batch)]
        if depth == 2:
            self.sets.append(self._second_set(layers_dev, outs_dev, in_groups, out_groups, engine.batch))
        self.s_in = torch.cuda.Stream()
        self.s_out = torch.cuda.Stream()
        self.s_desc = torch.cuda.Stream()
        self.ev_host = torch.cuda.Event()
        self.steps = 0

    @staticmethod
    def _new_set(layers_dev, outs_dev, in_groups, out_groups, batch):
        return {"layers": layers_dev, "outs": outs_dev, "in": in_groups, "out": out_groups, "batch": batch,
                "ev_in": [torch.cuda.Event() for _ in in_groups],
                "ev_used": [torch.cuda.Event() for _ in in_groups],    # the group's inputs are read
                "ev_done": [torch.cuda.Event() for _ in out_groups],   # the group's outputs are written
                "ev_out": [torch.cuda.Event() for _ in out_groups],    # the group's outputs have left
                "ev_desc": torch.cuda.Event(), "ev_step": torch.cuda.Event(), "used": False}

    @classmethod
    def _second_set(cls, layers_dev, outs_dev, in_groups, out_groups, batch):
        """Device buffers like the first set's (views at the same offsets of
        new group buffers) and a second device copy of the batch descriptors."""
        def twin(groups, tensors_of):
            new_groups, remap = [], {}
            for host, dev, idx in groups:
                if isinstance(dev, (tuple, list)):
                    dev2 = tuple(torch.empty_like(t) for t in dev)
                    for t, t2 in zip(dev, dev2):
                        remap[t.data_ptr()] = t2
                else:
                    dev2 = torch.empty_like(dev)
                    for i in idx:
                        for t in tensors_of(i):
                            off = t.data_ptr() - dev.data_ptr()
                            nb = t.numel() * t.element_size()
                            remap[t.data_ptr()] = dev2[off:off + nb].view(t.dtype).view(t.shape)
                new_groups.append((host, dev2, idx))
            return new_groups, remap
        in2, rin = twin(in_groups, lambda i: layers_dev[i][1:])
        out2, rout = twin(out_groups, lambda i: (outs_dev[i],))
        layers2 = [(l[0],) + tuple(rin[t.data_ptr()] for t in l[1:]) for l in layers_dev]
        outs2 = [rout[o.data_ptr()] for o in outs_dev]
        return cls._new_set(layers2, outs2, in2, out2, Batch(*batch.host, device=batch.dev[0].device))

    @staticmethod
    def _copy(dst, src):
        if isinstance(src, (tuple, list)):
            for d, s_ in zip(dst, src):
                d.copy_(s_, non_blocking=True)
        else:
            dst.copy_(src, non_blocking=True)

    def __call__(self):
        cur = torch.cuda.current_stream()
        st = self.sets[self.steps % len(self.sets)]
        n = len(st["layers"])
        if self.steps == 0:
            # the first step's copies begin after everything the caller queued
            # before it; later steps are ordered by the events below alone
            self.s_in.wait_stream(cur)
            self.s_desc.wait_stream(cur)
        if self.batch_host is not None:
            # the batch descriptors on their own stream: they wait for the end
            # of the last step that used this set, the layers' inputs only for
            # their buffers
            with torch.cuda.stream(self.s_desc):
                if st["used"]:
                    self.s_desc.wait_event(st["ev_step"])
                for t, dt in zip(self.batch_host, st["batch"].dev):
                    if t.numel():
                        dt[: t.numel()].copy_(t, non_blocking=True)
                st["ev_desc"].record(self.s_desc)
        with torch.cuda.stream(self.s_in):
            for g, (host, dev, _) in enumerate(st["in"]):
                if st["used"]:
                    self.s_in.wait_event(st["ev_used"][g])   # the last step of this set has read this group
                self._copy(dev, host)
                st["ev_in"][g].record(self.s_in)
        if self.batch_host is not None:
            cur.wait_event(st["ev_desc"])
        self.eng.batch = st["batch"]
        for i in range(n):
            layer, q, kq, vq = st["layers"][i]
            if i in self.in_first:
                cur.wait_event(st["ev_in"][self.in_first[i]])
            if st["used"] and i in self.out_first:
                cur.wait_event(st["ev_out"][self.out_first[i]])   # that step's O of the group has left
            self.eng.attend(layer, q, kq, vq, with_impact=(layer == self.impact_layer), o=st["outs"][i])
            if i in self.in_last:
                st["ev_used"][self.in_last[i]].record(cur)
            if i in self.out_last:
                g = self.out_last[i]
                st["ev_done"][g].record(cur)
                host, dev, _ = st["out"][g]
                with torch.cuda.stream(self.s_out):
                    self.s_out.wait_event(st["ev_done"][g])
                    self._copy(host, dev)
                    st["ev_out"][g].record(self.s_out)
        if self.impact_layer is not None:
            if self.steps > 0:
                cur.wait_event(self.ev_host)   # the previous step's top-k has left
            self.eng.select()
        st["ev_step"].record(cur)
        with torch.cuda.stream(self.s_out):
            self.s_out.wait_event(st["ev_step"])
            if self.impact_layer is not None and self.host_topk is not None:
                self.host_topk.copy_(self.eng.topk_idx, non_blocking=True)
            self.ev_host.record(self.s_out)
        st["used"] = True
        self.steps += 1

    def host_ready(self) -> torch.cuda.Event:
        """Event after the last device -> host copy of the latest step."""
        return self.ev_host
