"""Pins of the selective-recompute oracle (oracle/recompute.py) against facts
fixed outside it: the dense projection of a linear layer (torch), the page
geometry expanded token by token, and the invariants of copy on write.
A mutation test plants a wrong slot in the oracle and checks a pin fails."""

import struct

import numpy as np
import pytest
import torch

import oracle.prefill as orc
import oracle.recompute as rc
from workloads import get_workload, make_layer_inputs, make_layout, scaled

PAGE = 16


def small_case(seed=0):
    """Two requests that share a chunk, small heads, plus inputs of one layer."""
    w = scaled(get_workload("batched16"), num_q_heads=4, num_kv_heads=2, head_dim=16, n_requests=3,
               n_pool_chunks=4, chunk_len_range=(5, 70), chunks_per_req=(2, 3), q_range=(1, 4), d_model=48,
               seed=2000 + seed)
    lay = make_layout(w)
    inp = make_layer_inputs(w, lay, 0)
    g = torch.Generator().manual_seed(77 + seed)
    x = torch.randn(lay.total_doc, w.d_model, generator=g).to(torch.bfloat16)
    wk = (torch.randn(w.num_kv_heads * w.head_dim, w.d_model, generator=g) / 7).to(torch.bfloat16)
    wv = (torch.randn(w.num_kv_heads * w.head_dim, w.d_model, generator=g) / 7).to(torch.bfloat16)
    return w, lay, inp, x, wk, wv


def pools(w, lay, inp, spare):
    pk, pv = orc.build_layer_pool(lay, inp, np.uint16)
    grow = lambda p: np.concatenate([p, np.zeros((1, spare) + p.shape[2:], dtype=p.dtype)], axis=1)
    return grow(pk), grow(pv)


def request_chunks(lay, b, page_ids):
    """(page ids, length) per chunk-list entry of request b, from a page table."""
    out = []
    for e in range(int(lay.req_chunk_off[b]), int(lay.req_chunk_off[b + 1])):
        p0, p1 = int(lay.chunk_page_off[e]), int(lay.chunk_page_off[e + 1])
        out.append((np.asarray(page_ids[p0:p1]), int(lay.chunk_doc_off[e + 1] - lay.chunk_doc_off[e])))
    return out


def run(lay, selected, x, wk, wv, pk, pv, free, by_selection=False):
    p = rc.plan(lay.req_chunk_off, lay.chunk_doc_off, lay.chunk_page_off, lay.page_ids, selected, free,
                x_by_selection=by_selection)
    if by_selection:
        doc0 = lay.chunk_doc_off[lay.req_chunk_off[:-1]].tolist()
        rows = [doc0[b] + i for b in range(len(selected)) for i in selected[b]]
        xs = orc.to_f64(x)[rows] if rows else np.zeros((0, x.shape[1]))
    else:
        xs = orc.to_f64(x)
    if p.n_needed <= len(free):
        rc.apply(pk, pv, 0, p, xs, orc.to_f64(wk), orc.to_f64(wv))
    return p


def dense_projection_bits(x, wk):
    """bf16(x W^T), computed by torch's linear layer in fp64 (a library routine)."""
    y = torch.nn.functional.linear(x.to(torch.float64), wk.to(torch.float64))
    return y.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def dense_projection_v_bits(x, wv):
    """fp16(x W^T), V's stored type: torch's linear layer in fp64, rounded once
    to binary16 by Python's struct packing (torch's own fp64 -> fp16 goes
    through fp32 and rounds twice; the values here are far inside the range)."""
    y = torch.nn.functional.linear(x.to(torch.float64), wv.to(torch.float64)).numpy()
    flat = struct.pack(f"<{y.size}e", *y.ravel().tolist())
    return np.frombuffer(flat, dtype=np.uint16).reshape(y.shape)


def token_table(lay, b):
    """(page ref, slot) of every doc position of request b, expanded page by page."""
    out = []
    for e in range(int(lay.req_chunk_off[b]), int(lay.req_chunk_off[b + 1])):
        n = int(lay.chunk_doc_off[e + 1] - lay.chunk_doc_off[e])
        ref0 = int(lay.chunk_page_off[e])
        slots = [(ref0 + j, s) for j in range(-(-n // PAGE)) for s in range(PAGE)]
        out.extend(slots[:n])
    return out


def test_recomputing_every_token_gives_the_dense_projection():
    w, lay, inp, x, wk, wv = small_case()
    pk, pv = pools(w, lay, inp, spare=lay.page_ids.numel())
    free = np.arange(lay.num_pages, lay.num_pages + lay.page_ids.numel())
    selected = [list(range(n)) for n in lay.doc_lens]
    p = run(lay, selected, x, wk, wv, pk, pv, free)
    kd, vd = dense_projection_bits(x, wk), dense_projection_v_bits(x, wv)
    at = 0
    for b in range(lay.num_requests):
        n = lay.doc_lens[b]
        got_k = orc.gather(pk, 0, request_chunks(lay, b, p.new_page_ids)).reshape(n, -1)
        got_v = orc.gather(pv, 0, request_chunks(lay, b, p.new_page_ids)).reshape(n, -1)
        assert np.array_equal(got_k, kd[at:at + n]) and np.array_equal(got_v, vd[at:at + n])
        at += n
    # every page reference holds a selected token, so every one was copied
    assert p.n_needed == lay.page_ids.numel()
    assert sorted(p.new_page_ids.tolist()) == free.tolist()


def test_empty_selection_changes_nothing():
    w, lay, inp, x, wk, wv = small_case()
    pk, pv = pools(w, lay, inp, spare=8)
    k0, v0 = pk.copy(), pv.copy()
    p = run(lay, [[] for _ in range(lay.num_requests)], x, wk, wv, pk, pv, np.arange(lay.num_pages, lay.num_pages + 8))
    assert np.array_equal(p.new_page_ids, lay.page_ids.numpy())
    assert p.n_needed == 0 and len(p.cow_src) == 0 and len(p.x_row) == 0
    assert np.array_equal(pk, k0) and np.array_equal(pv, v0)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_copy_on_write_invariants(seed):
    w, lay, inp, x, wk, wv = small_case(seed)
    rng = np.random.default_rng(seed)
    selected = [sorted(rng.choice(n, size=max(1, n // 7), replace=False).tolist()) for n in lay.doc_lens]
    spare = lay.page_ids.numel()
    pk, pv = pools(w, lay, inp, spare)
    k0, v0 = pk.copy(), pv.copy()
    free = np.arange(lay.num_pages, lay.num_pages + spare)[::-1].copy()    # any order of free ids
    p = run(lay, selected, x, wk, wv, pk, pv, free)
    # the shared pages themselves are never written
    assert np.array_equal(pk[:, :lay.num_pages], k0[:, :lay.num_pages])
    assert np.array_equal(pv[:, :lay.num_pages], v0[:, :lay.num_pages])
    # dirty references, expanded token by token, get the first free ids in ascending reference order
    dirty = sorted({token_table(lay, b)[i][0] for b in range(lay.num_requests) for i in selected[b]})
    assert p.n_needed == len(dirty)
    for n, ref in enumerate(dirty):
        assert p.new_page_ids[ref] == free[n] and p.cow_src[n] == lay.page_ids[ref]
    clean = [r for r in range(lay.page_ids.numel()) if r not in set(dirty)]
    assert np.array_equal(p.new_page_ids[clean], lay.page_ids.numpy()[clean])
    kd, vd = dense_projection_bits(x, wk), dense_projection_v_bits(x, wv)
    doc0 = 0
    for b in range(lay.num_requests):
        table = token_table(lay, b)
        sel = set(selected[b])
        for i, (ref, slot) in enumerate(table):
            new, old = p.new_page_ids[ref], lay.page_ids[ref]
            want_k = kd[doc0 + i].reshape(w.num_kv_heads, w.head_dim) if i in sel else k0[0, old, :, slot]
            want_v = vd[doc0 + i].reshape(w.num_kv_heads, w.head_dim) if i in sel else v0[0, old, :, slot]
            assert np.array_equal(pk[0, new, :, slot], want_k) and np.array_equal(pv[0, new, :, slot], want_v)
        doc0 += lay.doc_lens[b]
    # a request's view is the original one except at its own selected tokens
    for b in range(lay.num_requests):
        before = orc.gather(k0, 0, request_chunks(lay, b, lay.page_ids.numpy()))
        after = orc.gather(pk, 0, request_chunks(lay, b, p.new_page_ids))
        keep = [i for i in range(lay.doc_lens[b]) if i not in set(selected[b])]
        assert np.array_equal(before[keep], after[keep])


def test_selection_order_rows_equal_doc_rows():
    w, lay, inp, x, wk, wv = small_case(1)
    selected = [[3, 0, 11], [7], [1, 2]][: lay.num_requests]
    free = np.arange(lay.num_pages, lay.num_pages + 10)
    a_k, a_v = pools(w, lay, inp, 10)
    b_k, b_v = pools(w, lay, inp, 10)
    run(lay, selected, x, wk, wv, a_k, a_v, free)
    run(lay, selected, x, wk, wv, b_k, b_v, free, by_selection=True)
    assert np.array_equal(a_k, b_k) and np.array_equal(a_v, b_v)


def test_too_few_free_pages_does_nothing():
    w, lay, inp, x, wk, wv = small_case()
    pk, pv = pools(w, lay, inp, 2)
    k0 = pk.copy()
    # the first token of every page
    selected = [[i for i, (_, slot) in enumerate(token_table(lay, b)) if slot == 0] for b in range(lay.num_requests)]
    p = run(lay, selected, x, wk, wv, pk, pv, np.arange(lay.num_pages, lay.num_pages + 2))
    assert p.n_needed == lay.page_ids.numel() > 2
    assert np.array_equal(p.new_page_ids, lay.page_ids.numpy()) and np.array_equal(pk, k0)


def test_mutation_wrong_slot_is_caught(monkeypatch):
    w, lay, inp, x, wk, wv = small_case()
    real = rc.locate

    def off_by_one(*a):
        ref, slot = real(*a)
        return ref, (slot + 1) % PAGE

    monkeypatch.setattr(rc, "locate", off_by_one)
    with pytest.raises(AssertionError):
        test_recomputing_every_token_gives_the_dense_projection()
