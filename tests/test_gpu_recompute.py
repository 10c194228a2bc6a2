"""Selective recompute on the GPU (plan, page copies, tcgen05 projection),
through the C ABI, against the oracle of oracle/recompute.py.

The selections are seeded draws, or the oracle's own top-k, never the GPU's
output. Integer work (the rewritten page table, the private pages, the copied
slots, every page the recompute must not touch) is compared bit for bit; the
recomputed rows are bf16(x W^T) on both sides, the GPU's from an fp32
accumulation, so a row element may differ by one bf16 rounding step:
|got - ref| <= 2^-7 |ref| + 1e-3.
"""

import numpy as np
import pytest
import torch

import oracle.prefill as orc
import oracle.recompute as orc_rc
from serving_prefill_b200 import Batch
from serving_prefill_b200.rag import (rag_recompute_kv, rag_recompute_plan, rag_recompute_plan_size,
                                      rag_recompute_status)
from workloads import get_workload, make_recompute_inputs, random_selection, scaled

from gpu_support import DeviceCase, assert_o_close

pytestmark = pytest.mark.gpu

RTOL = 2.0 ** -7
ATOL = 1e-3
RAG_ERR_NO_FREE_PAGES = 10


def cases():
    b16 = get_workload("batched16")
    l3 = get_workload("llama3_8b_l32")
    return {
        "pooled": scaled(b16, num_q_heads=8, num_kv_heads=2, n_requests=5, n_pool_chunks=10,
                         chunk_len_range=(1, 300), chunks_per_req=(1, 4), q_range=(1, 40), d_model=256),
        # several 128-token tiles of selected tokens with a ragged tail, a long K loop
        "tiles": scaled(l3, num_layers=2, num_q_heads=16, num_kv_heads=4, chunk_lens=(700, 333, 901), q_len=20,
                        d_model=1024),
        # an odd number of KV heads: output tiles of one head instead of two
        "odd_heads": scaled(b16, num_q_heads=6, num_kv_heads=3, n_requests=3, n_pool_chunks=6,
                            chunk_len_range=(20, 300), chunks_per_req=(1, 3), q_range=(1, 20), d_model=192),
    }


def to_bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def upload_selection(sel, device="cuda"):
    B = len(sel)
    k_cap = max(1, max(len(s) for s in sel))
    idx = torch.full((B, k_cap), -1, dtype=torch.int32)
    for b, s in enumerate(sel):
        idx[b, :len(s)] = torch.tensor(s, dtype=torch.int32)
    k = torch.tensor([len(s) for s in sel], dtype=torch.int32)
    return idx.to(device), k.to(device), k_cap


def run_case(w, sel, spare, layers=(0,), by_selection=False, free_order=None, v_scale=1.0):
    case = DeviceCase(w, layers=list(layers), spare_pages=spare)
    lay = case.lay
    free = np.arange(lay.num_pages, lay.num_pages + spare) if free_order is None else free_order
    idx, k, k_cap = upload_selection(sel)
    plan = torch.empty(rag_recompute_plan_size(case.batch, k_cap) // 4, dtype=torch.int32, device="cuda")
    page_out = torch.empty_like(case.batch.dev[3])
    free_dev = torch.tensor(free, dtype=torch.int32, device="cuda")
    rag_recompute_plan(case.batch, idx, k_cap, k, free_dev, page_out, plan, x_by_selection=by_selection)
    # oracle pools (this layer's bits), grown by the spare pages
    ref_plan = orc_rc.plan(lay.req_chunk_off, lay.chunk_doc_off, lay.chunk_page_off, lay.page_ids, sel, free,
                           x_by_selection=by_selection)
    results = []
    for layer in layers:
        rin = make_recompute_inputs(w, lay, layer)
        if v_scale != 1.0:   # V projections far beyond the fp16 range (both sides use these weights)
            rin.w_v = (rin.w_v.float() * v_scale).to(torch.bfloat16)
        if by_selection:
            doc0 = lay.chunk_doc_off[lay.req_chunk_off[:-1]].tolist()
            rows = [doc0[b] + i for b in range(len(sel)) for i in sel[b]]
            x = rin.x[rows] if rows else rin.x[:1]
        else:
            x = rin.x
        pk0 = to_bits(case.pool.k[layer])[None]
        pv0 = to_bits(case.pool.v[layer])[None]
        rag_recompute_kv(case.pool, layer, case.batch, k_cap, plan, x.cuda(), rin.w_k.cuda(), rin.w_v.cuda())
        torch.cuda.synchronize()
        ref_k, ref_v = pk0.copy(), pv0.copy()
        if ref_plan.n_needed <= len(free):
            orc_rc.apply(ref_k, ref_v, 0, ref_plan, orc.to_f64(x), orc.to_f64(rin.w_k), orc.to_f64(rin.w_v))
        results.append((layer, ref_k[0], ref_v[0], to_bits(case.pool.k[layer]), to_bits(case.pool.v[layer])))
    st, counts = rag_recompute_status(plan)
    return case, ref_plan, page_out.cpu().numpy(), st, counts, results


def assert_pool_matches(ref_plan, ref_bits, got_bits, decode, atol=None):
    """Bit-exact everywhere except the recomputed slots, which are within one
    bf16 step (decode: the stored format's values, bf16 for K, fp16 for V)."""
    sel = np.zeros(ref_bits.shape[:1] + ref_bits.shape[2:3], dtype=bool)   # [pages, slots]
    for page, slot in zip(ref_plan.dst_page, ref_plan.dst_slot):
        sel[page, slot] = True
    keep = ~sel
    assert np.array_equal(ref_bits.transpose(0, 2, 1, 3)[keep], got_bits.transpose(0, 2, 1, 3)[keep])
    if sel.any():
        r = decode(ref_bits.transpose(0, 2, 1, 3)[sel])
        g = decode(got_bits.transpose(0, 2, 1, 3)[sel])
        err = np.abs(g - r)
        bound = (ATOL if atol is None else atol) + RTOL * np.abs(r)
        assert (err <= bound).all(), f"recomputed rows: worst ratio {(err / bound).max():.3g}"


@pytest.mark.parametrize("name", ["pooled", "tiles", "odd_heads"])
@pytest.mark.parametrize("by_selection", [False, True])
def test_recompute_matches_oracle(name, by_selection):
    w = cases()[name]
    from workloads import make_layout
    lay = make_layout(w)
    counts = [orc.recompute_count(n, 0.15) for n in lay.doc_lens]
    sel = random_selection(lay.doc_lens, counts, seed=5)
    spare = lay.page_ids.numel()
    case, ref_plan, page_out, st, cnt, results = run_case(w, sel, spare, layers=range(w.num_layers),
                                                          by_selection=by_selection)
    assert st == 0, st
    assert np.array_equal(page_out, ref_plan.new_page_ids)
    assert cnt == (sum(len(s) for s in sel), len(ref_plan.cow_src), ref_plan.n_needed)
    for layer, rk, rv, gk, gv in results:
        assert_pool_matches(ref_plan, rk, gk, orc.bits_to_f64)
        assert_pool_matches(ref_plan, rv, gv, orc.f16_bits_to_f64)


def test_private_pages_come_from_the_free_list_in_reference_order():
    w = cases()["pooled"]
    from workloads import make_layout
    lay = make_layout(w)
    sel = random_selection(lay.doc_lens, [5] * lay.num_requests, seed=6)
    spare = lay.page_ids.numel()
    free = np.arange(lay.num_pages, lay.num_pages + spare)[::-1].copy()
    case, ref_plan, page_out, st, cnt, results = run_case(w, sel, spare, free_order=free)
    assert st == 0
    assert np.array_equal(page_out, ref_plan.new_page_ids)
    for layer, rk, rv, gk, gv in results:
        assert_pool_matches(ref_plan, rk, gk, orc.bits_to_f64)
        assert_pool_matches(ref_plan, rv, gv, orc.f16_bits_to_f64)


def test_too_few_free_pages_leaves_everything_unchanged():
    w = cases()["pooled"]
    from workloads import make_layout
    lay = make_layout(w)
    sel = [list(range(0, n, 9)) for n in lay.doc_lens]
    case, ref_plan, page_out, st, cnt, results = run_case(w, sel, spare=2)
    assert ref_plan.n_needed > 2
    assert st == RAG_ERR_NO_FREE_PAGES and cnt == (0, 0, ref_plan.n_needed)
    assert np.array_equal(page_out, lay.page_ids.numpy())
    for layer, rk, rv, gk, gv in results:
        assert np.array_equal(rk, gk) and np.array_equal(rv, gv)


def test_v_rows_beyond_the_fp16_range_are_saturated_and_reported():
    """V is stored as fp16: projected V values of magnitude ~2e5 saturate to
    65504 on both sides, and the plan's status reports RAG_ERR_RANGE. The
    absolute tolerance scales with the weights: an fp32 sum of d_model terms of
    magnitude ~2e5 that cancel is off by ~0.4 (the same sum in fp32 on the CPU
    is too)."""
    w = cases()["tiles"]
    from workloads import make_layout
    lay = make_layout(w)
    counts = [orc.recompute_count(n, 0.15) for n in lay.doc_lens]
    sel = random_selection(lay.doc_lens, counts, seed=7)
    case, ref_plan, page_out, st, cnt, results = run_case(w, sel, lay.page_ids.numel(), v_scale=2.0e5)
    assert st == 9, st   # RAG_ERR_RANGE
    for layer, rk, rv, gk, gv in results:
        assert_pool_matches(ref_plan, rk, gk, orc.bits_to_f64)
        assert_pool_matches(ref_plan, rv, gv, orc.f16_bits_to_f64, atol=ATOL * 2.0e5)
        assert (gv == 0x7BFF).any() and (gv == 0xFBFF).any()


def test_attention_after_recompute_uses_the_private_pages():
    """Top-k by the oracle, recompute on both sides, then attention over the
    rewritten page table: the GPU result matches the oracle's attention over
    the oracle's recomputed pool."""
    w = cases()["pooled"]
    from workloads import make_layout
    lay = make_layout(w)
    spare = lay.page_ids.numel()
    case0 = DeviceCase(w, layers=[0])
    ref0 = case0.oracle(0, True)
    sel = [t.tolist() for t in ref0.topk]
    case, ref_plan, page_out, st, cnt, results = run_case(w, sel, spare)
    assert st == 0
    # attention through the rewritten page table
    arrays = [lay.req_chunk_off, lay.chunk_doc_off, lay.chunk_page_off, torch.from_numpy(page_out), lay.q_off]
    batch = Batch(*arrays, device="cuda")
    from serving_prefill_b200.engine import PrefillEngine
    eng = PrefillEngine(case.pool, batch, w.num_q_heads, w.r, device="cuda")
    q, kq, vq = case.dev_inputs[0]
    eng.attend(0, q, kq, vq, with_impact=False)
    torch.cuda.synchronize()
    got = eng.o[: batch.total_q].float().cpu().double().numpy()
    # oracle attention over its own recomputed pool
    _, rk, rv, _, _ = results[0]
    inp = case.inputs[0]
    q_all, kq_all = orc.to_f64(inp.q), orc.to_f64(inp.kq)
    vq_all = orc.v_values(orc.v_operand_bits(orc.to_bits(inp.vq)))
    o_ref = np.zeros_like(got)
    q0 = 0
    for b, cs in enumerate(lay.req_chunks):
        ql = lay.q_lens[b]
        chunks = []
        for e in range(int(lay.req_chunk_off[b]), int(lay.req_chunk_off[b + 1])):
            p0, p1 = int(lay.chunk_page_off[e]), int(lay.chunk_page_off[e + 1])
            chunks.append((ref_plan.new_page_ids[p0:p1], int(lay.chunk_doc_off[e + 1] - lay.chunk_doc_off[e])))
        kd = orc.bits_to_f64(orc.gather(rk[None], 0, chunks))
        vd = orc.v_values(orc.gather(rv[None], 0, chunks))
        kcat = np.concatenate([kd, kq_all[q0:q0 + ql]])
        vcat = np.concatenate([vd, vq_all[q0:q0 + ql]])
        o, _, _, _, _ = orc.attend_request(q_all[q0:q0 + ql], kcat, vcat, kd.shape[0], 1 / np.sqrt(w.head_dim),
                                           want_impact=False)
        o_ref[q0:q0 + ql] = o
        q0 += ql
    assert_o_close(got, o_ref, "bf16")
