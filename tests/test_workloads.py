"""The seeded workload recipes: layout invariants the kernels and the oracle rely on."""

import numpy as np
import torch

import oracle.prefill as orc
from workloads import PAGE_SIZE, get_workload, make_layer_inputs, make_layout, scaled


def test_decode_layout_has_private_context_and_one_token():
    w = get_workload("decode16")
    lay = make_layout(w)
    assert lay.num_requests == w.n_requests
    assert lay.q_lens == [1] * w.n_requests
    tails = [cs[-1] for cs in lay.req_chunks]
    assert len(set(tails)) == len(tails), "every request owns its context chunk"
    shared = {c for cs in lay.req_chunks for c in cs[:-1]}
    assert not shared & set(tails), "a context chunk is never retrieved by another request"
    lo, hi = w.context_range
    assert all(lo <= lay.chunk_len[c] <= hi for c in tails)
    assert all(w.chunks_per_req[0] <= len(cs) - 1 <= w.chunks_per_req[1] for cs in lay.req_chunks)
    # pages: one per 16 tokens of every distinct chunk, all distinct
    pages = torch.cat(lay.chunk_pages).tolist()
    assert len(pages) == len(set(pages)) == lay.num_pages
    assert all(len(p) == -(-n // PAGE_SIZE) for p, n in zip(lay.chunk_pages, lay.chunk_len))


def test_prefill_layouts_are_unchanged_by_the_decode_fields():
    # the decode draw happens after every other draw, so the other recipes keep their layouts
    lay = make_layout(get_workload("batched16"))
    assert all(q >= 32 for q in lay.q_lens)
    assert len(lay.chunk_len) == 256


def test_one_token_query_is_unmasked_attention_over_every_key():
    # a decode step: the single query token sits after every cached key, so the
    # oracle's causal rule leaves nothing masked; compare with fp64 SDPA, no mask
    w = scaled(get_workload("decode16"), num_q_heads=4, num_kv_heads=2, n_requests=3, n_pool_chunks=5,
               chunk_len_range=(3, 40), chunks_per_req=(1, 3), context_range=(1, 30))
    lay = make_layout(w)
    inp = make_layer_inputs(w, lay, 0)
    res = orc.run_workload_layer(lay, inp, want_impact=False)
    q_all = orc.to_f64(inp.q)
    q0 = 0
    for b, cs in enumerate(lay.req_chunks):
        kd = np.concatenate([orc.to_f64(inp.chunk_k[c]) for c in cs] + [orc.to_f64(inp.kq[q0:q0 + 1])])
        vd = np.concatenate([orc.to_f64(inp.chunk_v[c]) for c in cs] + [orc.to_f64(inp.vq[q0:q0 + 1])])
        for h in range(w.num_q_heads):
            g = h // w.group
            q = torch.from_numpy(q_all[q0:q0 + 1, h][None, None])
            k = torch.from_numpy(kd[:, g][None, None])
            v = torch.from_numpy(vd[:, g][None, None])
            want = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=1.0 / np.sqrt(w.head_dim))
            np.testing.assert_allclose(res.o[q0, h], want[0, 0, 0].numpy(), rtol=1e-12, atol=1e-12)
        q0 += 1


def test_roofline_numerators_match_the_counts_by_hand():
    # bench.step_work feeds roofline.achieved; pin it to the counts worked out by
    # hand from each workload's shape (one QK^T and one PV per visible pair,
    # K and V of every doc token once per request)
    import sys, os
    sys.path.insert(0, os.path.abspath(os.path.join(os.path.dirname(__file__), "..")))
    import bench
    w = get_workload("llama2_7b_l1")
    work = bench.step_work(w, make_layout(w))
    pairs = 64 * 2048 + 64 * 65 // 2                      # doc keys for every row, causal inside the query
    assert work["attn_flops_per_launch"] == 4 * 128 * 32 * pairs
    assert abs(work["attn_flops_per_launch"] - 2.18e9) / 2.18e9 < 0.01
    kv = 2 * 2048 * 32 * 128 * 2                           # K and V, bf16
    assert abs(kv - 33.5e6) / 33.5e6 < 0.01
    assert work["attn_bytes_per_launch"] == kv + 64 * (32 + 2 * 32) * 128 * 2 + 64 * 32 * 128 * 2
    w70 = get_workload("long70b")
    work70 = bench.step_work(w70, make_layout(w70))
    pairs70 = 256 * 65536 + 256 * 257 // 2
    assert work70["attn_flops_per_launch"] == 4 * 128 * 64 * pairs70
    assert abs(work70["attn_flops_per_launch"] - 551e9) / 551e9 < 0.01
    assert abs(2 * 65536 * 8 * 128 * 2 - 268e6) / 268e6 < 0.01
