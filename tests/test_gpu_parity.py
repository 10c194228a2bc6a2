"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Sizes span several 128-key tiles, several 128-row tiles, ragged chunk tails,
several requests (up to 130), GQA groups of 1 to 8, split and unsplit key ranges, and the
edge cases of the method (one query token, one-token chunks, a request with
no query tokens, repeated chunks). The full-size workloads run in the launch
configuration the benchmark times.
"""

import numpy as np
import pytest
import torch

import oracle.prefill as orc
from workloads import get_workload, make_layout, scaled

from gpu_support import DeviceCase, assert_impact_close, check_layer

pytestmark = pytest.mark.gpu


def small_cases():
    l2 = get_workload("llama2_7b_l1")
    l3 = get_workload("llama3_8b_l32")
    b16 = get_workload("batched16")
    l70 = get_workload("long70b")
    return {
        "tiny": get_workload("tiny"),
        "tiny_f32_gqa": scaled(get_workload("tiny"), num_q_heads=8, num_kv_heads=2, head_dim=128,
                               chunk_lens=(33, 1, 16, 70), q_len=13),
        "mha_ragged": scaled(l2, num_q_heads=4, num_kv_heads=4, chunk_lens=(200, 77, 300), q_len=40),
        "gqa4_rows3": scaled(l3, num_layers=2, num_q_heads=16, num_kv_heads=4,
                             chunk_lens=(333, 129, 500, 17), q_len=70),
        "pooled": scaled(b16, num_q_heads=8, num_kv_heads=2, n_requests=5, n_pool_chunks=12,
                         chunk_len_range=(1, 400), chunks_per_req=(1, 4), q_range=(1, 90)),
        "g8_long_rows": scaled(l70, num_q_heads=16, num_kv_heads=2, chunk_lens=(700,) * 6, q_len=150),
        "decode": scaled(get_workload("decode16"), num_q_heads=8, num_kv_heads=2, n_requests=6, n_pool_chunks=10,
                         chunk_len_range=(1, 300), chunks_per_req=(1, 4), context_range=(1, 200)),
        "decode_mha": scaled(get_workload("decode16"), num_q_heads=4, num_kv_heads=4, n_requests=3, n_pool_chunks=6,
                             chunk_len_range=(1, 700), chunks_per_req=(1, 3), context_range=(1, 64)),
        "decode_g8_long": scaled(get_workload("decode16"), num_q_heads=16, num_kv_heads=2, n_requests=2,
                                 n_pool_chunks=4, chunk_len_range=(2000, 5000), chunks_per_req=(3, 4),
                                 context_range=(300, 400)),
        "one_query_token": scaled(l2, num_q_heads=8, num_kv_heads=8, chunk_lens=(1, 15, 16, 17, 129), q_len=1),
        "query_longer_than_tile": scaled(l3, num_layers=1, num_q_heads=4, num_kv_heads=2, chunk_lens=(60,),
                                         q_len=300),
        # query blocks of at most 16 rows take the decode kernel: 16 rows of
        # 4 causal query tokens, 10 rows of 5 tokens (padded to 16), and a
        # batch whose items pad to 4, 8 or 16 rows
        "short_query_g4": scaled(l3, num_layers=1, num_q_heads=8, num_kv_heads=2, chunk_lens=(300, 77, 1), q_len=4),
        "short_query_g2": scaled(l3, num_layers=1, num_q_heads=4, num_kv_heads=2, chunk_lens=(129, 16, 200), q_len=5),
        "short_queries_batched": scaled(b16, num_q_heads=8, num_kv_heads=2, n_requests=5, n_pool_chunks=6,
                                        chunk_len_range=(1, 300), chunks_per_req=(1, 3), q_range=(1, 4)),
        # many requests: one prefix entry per request in the kernels' shared memory
        "many_requests": scaled(b16, num_q_heads=8, num_kv_heads=2, n_requests=130, n_pool_chunks=40,
                                chunk_len_range=(1, 300), chunks_per_req=(1, 3), q_range=(1, 40)),
    }


CASES = small_cases()


@pytest.mark.parametrize("name", list(CASES))
def test_parity_small(name):
    w = CASES[name]
    layers = list(range(w.num_layers))
    case = DeviceCase(w, layers=layers)
    for layer in layers:
        check_layer(case, layer, with_impact=(layer == w.impact_layer_index))


def _keys_growing_by_chunk(inp):
    # chunk c's keys times 4^c (exact in bf16): along a request's keys the row
    # maxima jump by many 2^8 steps, so O is rescaled in the middle of rows
    for c, k in enumerate(inp.chunk_k):
        k.mul_(float(4 ** (c % 4)))


@pytest.mark.parametrize("name", ["decode_kernel", "prefill_kernel"])
def test_rescale_when_row_maxima_grow(name):
    w = {
        # 4 rows per unit: the decode kernel
        "decode_kernel": scaled(get_workload("decode16"), num_q_heads=8, num_kv_heads=2, n_requests=3, n_pool_chunks=4,
                                chunk_len_range=(150, 400), chunks_per_req=(3, 4), context_range=(1, 40)),
        # 80 rows per unit: the prefill kernel
        "prefill_kernel": scaled(get_workload("llama3_8b_l32"), num_layers=1, num_q_heads=8, num_kv_heads=2,
                                 chunk_lens=(200, 256, 300, 180), q_len=20),
    }[name]
    case = DeviceCase(w, layers=[0], transform=_keys_growing_by_chunk)
    check_layer(case, 0, with_impact=(w.impact_layer_index == 0))


@pytest.mark.parametrize("name", ["tiny", "pooled", "gqa4_rows3"])
def test_pool_write_bit_exact(name):
    w = CASES[name]
    case = DeviceCase(w, layers=[0])
    ref = orc.run_workload_layer(case.lay, case.inputs[0], want_impact=False, keep_pool=True)
    view = torch.int16 if w.dtype == "bf16" else torch.int32
    bits = np.uint16 if w.dtype == "bf16" else np.uint32
    gk = case.pool.k[0].contiguous().view(view).cpu().numpy().view(bits)
    gv = case.pool.v[0].contiguous().view(view).cpu().numpy().view(bits)
    assert np.array_equal(gk, ref.pool_k[0]) and np.array_equal(gv, ref.pool_v[0])
    assert int(case.err.item()) == 0


def test_physical_page_permutation_is_bit_identical():
    w = CASES["pooled"]
    lay = make_layout(w)
    a = DeviceCase(w, lay=lay, layers=[0]).run_layer(0, True)
    b = DeviceCase(w, lay=lay.with_page_permutation(seed=11), layers=[0]).run_layer(0, True)
    assert np.array_equal(a["o"], b["o"])
    assert np.array_equal(a["lse"], b["lse"])
    assert np.array_equal(a["topk_idx"], b["topk_idx"])
    np.testing.assert_allclose(a["impact"], b["impact"], rtol=1e-6)


def test_chunk_order_permutes_impact():
    w = CASES["mha_ragged"]
    lay = make_layout(w)
    order = [2, 0, 1]
    lay2 = lay.with_chunk_order([order])
    a = DeviceCase(w, lay=lay, layers=[0]).run_layer(0, True)
    b = DeviceCase(w, lay=lay2, layers=[0]).run_layer(0, True)
    np.testing.assert_allclose(a["o"], b["o"], atol=2e-2, rtol=2e-2)
    starts1 = np.cumsum([0] + [lay.chunk_len[c] for c in lay.req_chunks[0]])
    starts2 = np.cumsum([0] + [lay2.chunk_len[c] for c in lay2.req_chunks[0]])
    for pos2, c in enumerate(lay2.req_chunks[0]):
        pos1 = lay.req_chunks[0].index(c)
        n = lay.chunk_len[c]
        assert_impact_close(b["impact"][starts2[pos2]:starts2[pos2] + n], a["impact"][starts1[pos1]:starts1[pos1] + n])


def test_request_without_query_tokens():
    w = scaled(get_workload("batched16"), num_q_heads=8, num_kv_heads=2, n_requests=3, n_pool_chunks=5,
               chunk_len_range=(20, 200), chunks_per_req=(1, 3), q_range=(1, 40))
    lay = make_layout(w)
    lay.q_lens[1] = 0
    from workloads.rag import _flatten
    _flatten(lay)
    case = DeviceCase(w, lay=lay, layers=[0])
    out, ref = check_layer(case, 0, with_impact=True)
    n0 = lay.doc_lens[0] + lay.q_lens[0]
    assert np.all(out["impact"][n0:n0 + lay.doc_lens[1]] == 0)


def test_impact_total_is_query_length():
    w = CASES["pooled"]
    case = DeviceCase(w, layers=[0])
    out = case.run_layer(0, True)
    at = 0
    for b in range(case.lay.num_requests):
        n = case.lay.doc_lens[b] + case.lay.q_lens[b]
        np.testing.assert_allclose(out["impact"][at:at + n].sum(), case.lay.q_lens[b], rtol=1e-4)
        at += n


def test_run_twice_is_deterministic_for_o():
    w = CASES["g8_long_rows"]
    case = DeviceCase(w, layers=[0])
    a = case.run_layer(0, False)
    b = case.run_layer(0, False)
    assert np.array_equal(a["o"], b["o"]) and np.array_equal(a["lse"], b["lse"])


# ------------------------------------------------------------------ full size

@pytest.mark.slow
@pytest.mark.parametrize("name", ["tiny", "llama2_7b_l1", "batched16", "long70b"])
def test_parity_full_size(name):
    w = get_workload(name)
    case = DeviceCase(w, layers=[w.impact_layer_index])
    check_layer(case, w.impact_layer_index, with_impact=True)


@pytest.mark.slow
def test_parity_at_the_request_limit():
    """4,096 small requests, the most a batch may hold: prefixes, grids and the per-request top-k at full width."""
    w = scaled(get_workload("batched16"), name="requests_4096", num_q_heads=4, num_kv_heads=2, n_requests=4096,
               n_pool_chunks=64, chunk_len_range=(1, 40), chunks_per_req=(1, 2), q_range=(1, 3))
    case = DeviceCase(w, layers=[0])
    check_layer(case, 0, with_impact=True)


@pytest.mark.slow
def test_parity_full_size_decode():
    """One decode step of 16 requests: a new token over retrieved chunks and the request's own context."""
    w = get_workload("decode16")
    case = DeviceCase(w, layers=[0])
    check_layer(case, 0, with_impact=False)


@pytest.mark.slow
def test_parity_full_size_32_layers():
    """All 32 layers run as the benchmark runs them; layers 0 and 31 (impact) are checked."""
    w = get_workload("llama3_8b_l32")
    case = DeviceCase(w)
    for layer in range(w.num_layers):
        q, kq, vq = case.dev_inputs[layer]
        case.engine.attend(layer, q, kq, vq, with_impact=False)
    torch.cuda.synchronize()
    check_layer(case, 0, with_impact=False)
    check_layer(case, w.num_layers - 1, with_impact=True)


def test_host_step_matches_the_device_step():
    """The pipelined step from pinned host buffers (copies on their own
    streams, ordered by events) gives the same outputs as the plain step,
    twice in a row."""
    from serving_prefill_b200.engine import HostStep, layer_groups
    w = CASES["gqa4_rows3"]
    case = DeviceCase(w)
    layers = [(l,) + case.dev_inputs[l] for l in case.layers]
    outs = [torch.empty_like(case.engine.o) for _ in layers]
    case.engine.step(layers, w.impact_layer_index, outs=outs)
    torch.cuda.synchronize()
    want_o = [o.clone() for o in outs]
    want_idx = case.engine.topk_idx.clone()
    host_in = [tuple(t.cpu().pin_memory() for t in case.dev_inputs[l]) for l in case.layers]
    dev_in = [(l,) + tuple(torch.empty_like(t) for t in case.dev_inputs[l]) for l in case.layers]
    dev_out = [torch.empty_like(o) for o in outs]
    host_out = [torch.empty_like(o, device="cpu").pin_memory() for o in outs]
    host_topk = torch.empty_like(want_idx, device="cpu").pin_memory()
    desc = [t.contiguous().pin_memory() for t in case.batch.host]
    step = HostStep(case.engine, dev_in, dev_out, host_in, host_out, w.impact_layer_index, host_topk=host_topk,
                    batch_host=desc)
    # the same step with every layer's inputs, and every layer's O, moved as one group
    in_groups, _, gdev_in = layer_groups([case.dev_inputs[l] for l in case.layers], len(layers), "cuda")
    out_groups, gout_host, gout_dev = layer_groups([(o,) for o in outs], len(layers), "cuda", fill=False)
    gstep = HostStep(case.engine, [(l,) + gdev_in[n] for n, l in enumerate(case.layers)], [v[0] for v in gout_dev],
                     None, None, w.impact_layer_index, host_topk=host_topk, batch_host=desc, in_groups=in_groups,
                     out_groups=out_groups)
    # and two-deep: consecutive steps alternate between two device buffer sets
    dstep = HostStep(case.engine, [(l,) + gdev_in[n] for n, l in enumerate(case.layers)], [v[0] for v in gout_dev],
                     None, None, w.impact_layer_index, host_topk=host_topk, batch_host=desc, in_groups=in_groups,
                     out_groups=out_groups, depth=2)
    for run, got in ([(step, host_out)] * 2 + [(gstep, [v[0] for v in gout_host])] * 2 +
                     [(dstep, [v[0] for v in gout_host])] * 3):
        run()
        torch.cuda.synchronize()
        for a, b in zip(got, want_o):
            assert torch.equal(a[: case.batch.total_q], b[: case.batch.total_q].cpu())   # O is run-to-run stable
        # the selection that came back is the one on the device (Impact sums by
        # atomics, so near-ties may order differently from the first run)
        assert torch.equal(host_topk, case.engine.topk_idx.cpu())
