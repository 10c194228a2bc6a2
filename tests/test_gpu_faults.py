"""Failure detection on the GPU, with every fault made on the host.

Bad descriptors are injected into the batch the host passes (a page id outside
the pool, a chunk with one page too many or too few) and an out-of-range V
value into the pool; the kernels skip or mask what they cannot use, record it
in the workspace error word, and the call returns. A self-test kernel runs the
bounded mbarrier wait every pipeline uses until it gives up. Nothing here
faults, traps or hangs the GPU: the TMA boxes of a bad page are requested at a
negative row, which the copy engine fills with zeros, and every wait has a
limit.
"""

import numpy as np
import pytest
import torch

import oracle.prefill as orc
from serving_prefill_b200 import Batch, rag_last_device_error
from serving_prefill_b200.engine import PrefillEngine
from serving_prefill_b200.rag import rag_kv_pool_write, rag_selftest_wait_timeout
from workloads import get_workload, make_layout, scaled

from gpu_support import DeviceCase, assert_impact_close, assert_o_close, check_layer

pytestmark = pytest.mark.gpu

RAG_ERR_PAGE_OOB, RAG_ERR_TIMEOUT, RAG_ERR_GEOMETRY, RAG_ERR_RANGE = 3, 6, 8, 9


def pooled(path="prefill"):
    """Four requests over a shared chunk pool; path "decode" gives them 1-4
    query tokens (at most 16 rows per unit), so the decode kernel runs."""
    q_range = (1, 4) if path == "decode" else (5, 60)
    return scaled(get_workload("batched16"), num_q_heads=8, num_kv_heads=2, n_requests=4, n_pool_chunks=8,
                  chunk_len_range=(20, 300), chunks_per_req=(2, 3), q_range=q_range)


PATHS = ["prefill", "decode"]


def host_arrays(lay):
    return [t.clone() for t in (lay.req_chunk_off, lay.chunk_doc_off, lay.chunk_page_off, lay.page_ids, lay.q_off)]


def run_with_batch(case, arrays):
    """Run the layer with another batch descriptor over the same pool and inputs."""
    batch = Batch(*arrays, device="cuda")
    eng = PrefillEngine(case.pool, batch, case.w.num_q_heads, case.w.r, device="cuda")
    eng.o.zero_()
    q, kq, vq = case.dev_inputs[0]
    eng.attend(0, q, kq, vq, with_impact=True)
    eng.select()
    torch.cuda.synchronize()
    st, bits = rag_last_device_error(eng.ws)
    out = {"o": eng.o[: batch.total_q].float().cpu().double().numpy(),
           "impact": eng.impact[: batch.total_doc + batch.total_q].cpu().double().numpy(),
           "topk_idx": eng.topk_idx.cpu().numpy(), "k": eng.k.cpu().numpy()}
    return st, bits, out


def check_other_requests(case, out, ref, skip):
    """Every request except `skip` matches the oracle."""
    lay = case.lay
    q0 = at = 0
    for b in range(lay.num_requests):
        ql, nd = lay.q_lens[b], lay.doc_lens[b]
        if b != skip:
            assert_o_close(out["o"][q0:q0 + ql], ref.o[q0:q0 + ql], "bf16")
            assert_impact_close(out["impact"][at:at + nd + ql], ref.impact[at:at + nd + ql])
            assert int(out["k"][b]) == ref.k[b]
        q0 += ql
        at += nd + ql


@pytest.mark.parametrize("path", PATHS)
def test_page_outside_the_pool_is_skipped_and_reported(path):
    w = pooled(path)
    case = DeviceCase(w, layers=[0])
    ref = case.oracle(0, True)
    arrays = host_arrays(case.lay)
    arrays[3][0] = case.lay.num_pages + 5            # request 0's first page
    st, bits, out = run_with_batch(case, arrays)
    assert st == RAG_ERR_PAGE_OOB and bits & 1, (st, bits)
    assert np.isfinite(out["o"]).all() and np.isfinite(out["impact"]).all()
    check_other_requests(case, out, ref, skip=0)
    # the missing page's 16 tokens are masked: no weight reaches them
    assert np.all(out["impact"][:16] == 0)
    k0 = int(out["k"][0])
    assert len(set(out["topk_idx"][0][:k0].tolist())) == k0


@pytest.mark.parametrize("path", PATHS)
def test_chunk_with_one_page_too_many_is_reported_and_exact(path):
    w = pooled(path)
    case = DeviceCase(w, layers=[0])
    ref = case.oracle(0, True)
    rc, cd, cp, pid, qo = host_arrays(case.lay)
    c = 0                                             # request 0's first chunk-list entry
    extra = int(pid[-1])                              # a valid page id: never read, its slots are masked
    end = int(cp[c + 1])
    pid = torch.cat([pid[:end], torch.tensor([extra], dtype=torch.int32), pid[end:]])
    cp = cp.clone()
    cp[c + 1:] += 1
    st, bits, out = run_with_batch(case, [rc, cd, cp, pid, qo])
    assert st == RAG_ERR_GEOMETRY and bits == 2, (st, bits)
    check_other_requests(case, out, ref, skip=-1)    # every request, the altered one included


@pytest.mark.parametrize("path", PATHS)
def test_chunk_with_one_page_too_few_is_reported(path):
    w = pooled(path)
    case = DeviceCase(w, layers=[0])
    ref = case.oracle(0, True)
    rc, cd, cp, pid, qo = host_arrays(case.lay)
    lens = (cd[1:] - cd[:-1]).tolist()
    # the request with the fewest doc tokens, so that the batch's host maxima
    # (which the host checks before launching) come from another request
    bad = int(np.argmin(case.lay.doc_lens))
    c = next(i for i in range(int(rc[bad]), int(rc[bad + 1])) if lens[i] > 16)   # a chunk of two pages or more
    end = int(cp[c + 1])
    pid = torch.cat([pid[:end - 1], pid[end:]])
    cp = cp.clone()
    cp[c + 1:] -= 1
    st, bits, out = run_with_batch(case, [rc, cd, cp, pid, qo])
    assert st == RAG_ERR_GEOMETRY and bits & 2, (st, bits)
    assert np.isfinite(out["o"]).all() and np.isfinite(out["impact"]).all()
    check_other_requests(case, out, ref, skip=bad)


@pytest.mark.parametrize("value,flagged", [(65280.0, False), (70000.0, True), (float("inf"), True)])
def test_v_beyond_the_fp16_range_is_reported_by_the_pool_write(value, flagged):
    """A bf16 pool keeps V in fp16: 65,280 is exact there; 70,000 and inf
    saturate to 65,504 and the write reports RAG_ERR_RANGE's bit. The oracle
    stores V the same way, so attention keeps full parity either way."""
    w = scaled(get_workload("llama2_7b_l1"), num_q_heads=4, num_kv_heads=4, chunk_lens=(200, 77), q_len=20)
    case = DeviceCase(w, layers=[0])
    inp = case.inputs[0]
    inp.chunk_v[0][3, 1, 5] = value                  # one V value of chunk 0 (also the oracle's input)
    pages = case.lay.chunk_pages[0].to(torch.int32).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rag_kv_pool_write(case.pool, 0, pages, inp.chunk_k[0].cuda(), inp.chunk_v[0].cuda(), device_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == (8 if flagged else 0)
    stored = case.pool.v[0].float()
    assert stored.abs().max().item() <= 65504.0
    check_layer(case, 0, with_impact=True)


@pytest.mark.parametrize("path", PATHS)
def test_v_q_beyond_the_fp16_range_is_reported_by_the_attention(path):
    """The query block's own V_q enters the product as fp16 too: a value of
    70,000 is saturated and the call reports RAG_ERR_RANGE; the rest of the
    output keeps parity with the oracle, which saturates it the same way
    (a 4-token query block takes the decode kernel)."""
    q_len = 4 if path == "decode" else 20
    w = scaled(get_workload("llama2_7b_l1"), num_q_heads=4, num_kv_heads=4, chunk_lens=(200, 77), q_len=q_len)
    case = DeviceCase(w, layers=[0])
    inp = case.inputs[0]
    inp.vq[min(7, q_len - 1), 2, 100] = 70000.0
    case.dev_inputs[0] = (inp.q.cuda(), inp.kq.cuda(), inp.vq.cuda())
    out = case.run_layer(0, with_impact=True)
    ref = case.oracle(0, True)
    st, bits = case.engine.device_error()
    assert st == RAG_ERR_RANGE and bits == 8, (st, bits)
    assert_o_close(out["o"], ref.o, w.dtype)


def test_bounded_wait_gives_up_and_reports_a_timeout():
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    rag_selftest_wait_timeout(err, 1_000_000)       # 1 ms
    e1.record()
    torch.cuda.synchronize()
    assert int(err.item()) == 4
    # the second role left on the abort flag, long before its own 2 s limit
    assert e0.elapsed_time(e1) < 500.0
    # the context is still usable: a small case runs to parity afterwards
    w = pooled()
    case = DeviceCase(w, layers=[0])
    check_layer(case, 0, with_impact=True)
