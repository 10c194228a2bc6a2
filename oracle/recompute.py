"""Plain fp64 definition of selective KV recompute into copy-on-write pages.

TEST INFRASTRUCTURE: only the tests, the smoke check and the benchmark's
CPU-baseline leg use this module. It shares no code with the CUDA library and
imports nothing from it.

What it computes (CacheBlend page, "Contributions": only the tokens of high
attention impact are recomputed when the cached KV are fused; "How it works":
the flow goes concatenate -> pick high-Impact tokens -> recompute their KV
values -> generate from the fused cache):

1. Page plan. A selected token is a logical doc position i of request b
   (0 <= i < N_doc,b, as the top-k reports it). It lives in chunk-list entry e
   of the request (the entry whose doc range holds i), at offset t = i - start_e
   of that chunk, i.e. in page reference ref = page_off_e + t // 16, slot
   t % 16. A chunk's pages are shared by every request that retrieved the
   chunk, so the request never writes them: each page reference that holds at
   least one selected token gets a private copy (copy on write). The private
   pages come from a caller-given list of free page ids, handed out in
   ascending order of page reference over the whole batch. The request's page
   table is rewritten to point at its private pages; every other reference
   keeps its page.
2. Per layer: each private page first receives the whole content of the page
   it replaces (every KV head, all 16 slots, K and V); then every selected
   token's K and V rows are recomputed from its hidden state x (the layer's
   input for that token): K = x W_K^T, V = x W_V^T, with W_K, W_V of shape
   [H_kv * d, d_model] (a linear layer's weight), split into H_kv heads of d,
   rounded once to the type the pool stores it in (a bf16 cache keeps K in
   bf16 and V in fp16; round to nearest even, V saturated beyond 65504), and
   stored in the token's slot of its private page.

The hidden states are gathered per selected token either by its doc position
(row doc_start_b + i of a [total_doc, d_model] array) or by its rank in the
selection (row t of a [sum_b k_b, d_model] array, selection order). The pages'
listing stops at the selection, so this restatement fixes what the recompute
writes and where; the arithmetic is the projection itself.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from .prefill import f16_bits_sat

PAGE_SIZE = 16


@dataclass
class RecomputePlan:
    new_page_ids: np.ndarray     # [num_page_refs] the batch's page table after copy on write
    cow_src: np.ndarray          # [n_cow] page copied from
    cow_dst: np.ndarray          # [n_cow] private page copied to
    x_row: np.ndarray            # [T] row of the hidden-state array per selected token
    dst_page: np.ndarray         # [T] private page of each selected token
    dst_slot: np.ndarray         # [T] its slot
    n_needed: int                # private pages the selection needs


def locate(req_chunk_off, chunk_doc_off, chunk_page_off, b, pos):
    """Page reference and slot of logical doc position `pos` of request b."""
    c0, c1 = int(req_chunk_off[b]), int(req_chunk_off[b + 1])
    doc0 = int(chunk_doc_off[c0])
    for e in range(c0, c1):
        start = int(chunk_doc_off[e]) - doc0
        end = int(chunk_doc_off[e + 1]) - doc0
        if start <= pos < end:
            t = pos - start
            return int(chunk_page_off[e]) + t // PAGE_SIZE, t % PAGE_SIZE
    raise IndexError(f"position {pos} outside request {b}")


def plan(req_chunk_off, chunk_doc_off, chunk_page_off, page_ids, selected, free_pages,
         x_by_selection: bool = False) -> RecomputePlan:
    """Copy-on-write page plan for a batch.

    selected: per request, the list of selected logical doc positions (in the
    order the selection lists them). free_pages: caller-owned free page ids.
    When the selection needs more private pages than `free_pages` holds,
    nothing is remapped and nothing is recomputed (n_needed tells how many).
    """
    req_chunk_off = np.asarray(req_chunk_off, dtype=np.int64)
    chunk_doc_off = np.asarray(chunk_doc_off, dtype=np.int64)
    chunk_page_off = np.asarray(chunk_page_off, dtype=np.int64)
    page_ids = np.asarray(page_ids, dtype=np.int64)
    B = len(req_chunk_off) - 1
    where = []                      # (b, ref, slot, x row) per selected token, selection order
    t = 0
    for b in range(B):
        doc0 = int(chunk_doc_off[req_chunk_off[b]])
        for pos in selected[b]:
            ref, slot = locate(req_chunk_off, chunk_doc_off, chunk_page_off, b, int(pos))
            where.append((ref, slot, t if x_by_selection else doc0 + int(pos)))
            t += 1
    dirty = sorted({ref for ref, _, _ in where})
    n_needed = len(dirty)
    new_ids = page_ids.copy()
    if n_needed > len(free_pages):
        empty = np.zeros(0, dtype=np.int64)
        return RecomputePlan(new_ids, empty, empty, empty, empty, empty, n_needed)
    private = {ref: int(free_pages[n]) for n, ref in enumerate(dirty)}
    for ref, p in private.items():
        new_ids[ref] = p
    cow_src = np.array([page_ids[ref] for ref in dirty], dtype=np.int64)
    cow_dst = np.array([private[ref] for ref in dirty], dtype=np.int64)
    x_row = np.array([x for _, _, x in where], dtype=np.int64)
    dst_page = np.array([private[ref] for ref, _, _ in where], dtype=np.int64)
    dst_slot = np.array([s for _, s, _ in where], dtype=np.int64)
    return RecomputePlan(new_ids, cow_src, cow_dst, x_row, dst_page, dst_slot, n_needed)


def round_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp64 values -> bf16 bits, rounded once to nearest even."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def apply(pool_k: np.ndarray, pool_v: np.ndarray, layer: int, p: RecomputePlan, x: np.ndarray,
          w_k: np.ndarray, w_v: np.ndarray) -> None:
    """One layer of the recompute, in place on the pools [L][pages][H_kv][16][d]
    of a bf16 cache (K: bf16 bits, V: fp16 bits).

    x: hidden states (exact fp64 values of the bf16 inputs), rows as p.x_row
    names them; w_k, w_v: [H_kv * d, d_model] (fp64 values).
    """
    _, _, hk, _, d = pool_k.shape
    for src, dst in zip(p.cow_src, p.cow_dst):
        pool_k[layer, dst] = pool_k[layer, src]
        pool_v[layer, dst] = pool_v[layer, src]
    if len(p.x_row) == 0:
        return
    xs = x[p.x_row]                                   # gather: one hidden state per selected token
    k_new = round_bf16_bits(xs @ w_k.T).reshape(len(p.x_row), hk, d)
    v_new = f16_bits_sat(xs @ w_v.T).reshape(len(p.x_row), hk, d)
    for t in range(len(p.x_row)):
        pool_k[layer, p.dst_page[t], :, p.dst_slot[t], :] = k_new[t]
        pool_v[layer, p.dst_page[t], :, p.dst_slot[t], :] = v_new[t]
