"""Decode of quantized chunk caches into the pool on the GPU (rag_kv_decode),
bit for bit against the codec oracle (oracle/codec.py): the codes and scales
come from the oracle's encoder run on the seeded chunk caches; the GPU and the
oracle decode them into pools that start from the same sentinel pattern, and
the whole pools must be equal. Chunks of ragged lengths (one token, whole
pages, partial last pages), 8- and 4-bit codes, several KV heads."""

import numpy as np
import pytest
import torch

import oracle.codec as codec
import oracle.prefill as orc
from serving_prefill_b200 import KVPool
from serving_prefill_b200.rag import rag_kv_decode
from workloads import get_workload, make_layer_inputs, make_layout, scaled

pytestmark = pytest.mark.gpu

SENTINEL = 0x7FBF   # a bf16 NaN pattern no decode produces


def build(w, bits, layer=0):
    lay = make_layout(w)
    inp = make_layer_inputs(w, lay, layer)
    encs = [codec.encode(orc.to_f64(k), orc.to_f64(v), bits) for k, v in zip(inp.chunk_k, inp.chunk_v)]
    return lay, encs


def run(w, bits, layers=(0, 1), tweak=None):
    lay, _ = build(w, bits)
    L = max(layers) + 1
    pool = KVPool(L, lay.num_pages, w.num_kv_heads, w.head_dim, device="cuda")
    pool.k.view(torch.int16).fill_(SENTINEL - 65536 if SENTINEL > 32767 else SENTINEL)
    pool.v.view(torch.int16).copy_(pool.k.view(torch.int16))
    ref_k = np.full(tuple(pool.k.shape), SENTINEL, dtype=np.uint16)
    ref_v = ref_k.copy()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for layer in layers:
        _, encs = build(w, bits, layer)
        if tweak:
            tweak(encs)
        n = [lay.chunk_len[c] for c in range(len(encs))]
        tok_off = torch.tensor(np.cumsum([0] + n), dtype=torch.int32, device="cuda")
        page_off = torch.tensor(np.cumsum([0] + [len(p) for p in lay.chunk_pages]), dtype=torch.int32, device="cuda")
        pages = torch.cat(lay.chunk_pages).to(torch.int32).cuda()
        cat = lambda xs: torch.from_numpy(np.ascontiguousarray(np.concatenate(xs))).cuda()
        rag_kv_decode(pool, layer, tok_off, page_off, pages, bits, cat([e.codes_k for e in encs]),
                      cat([e.codes_v for e in encs]), cat([e.scale_k[None] for e in encs]),
                      cat([e.offset_k[None] for e in encs]), cat([e.scale_v[None] for e in encs]),
                      cat([e.offset_v[None] for e in encs]), device_err=err)
        for c, e in enumerate(encs):
            codec.decode_into_pool(ref_k, ref_v, layer, lay.chunk_pages[c].numpy(), e, n[c])
    torch.cuda.synchronize()
    got_k = pool.k.view(torch.int16).cpu().numpy().view(np.uint16)
    got_v = pool.v.view(torch.int16).cpu().numpy().view(np.uint16)
    return got_k, got_v, ref_k, ref_v, int(err.item())


def cases():
    return {
        "ragged": scaled(get_workload("llama3_8b_l32"), num_layers=2, num_q_heads=8, num_kv_heads=2,
                         chunk_lens=(1, 16, 33, 100, 255), q_len=4),
        "pooled": scaled(get_workload("batched16"), num_layers=2, num_q_heads=32, num_kv_heads=8,
                         n_requests=3, n_pool_chunks=7, chunk_len_range=(1, 300), chunks_per_req=(1, 3),
                         q_range=(1, 4)),
    }


@pytest.mark.parametrize("name", ["ragged", "pooled"])
@pytest.mark.parametrize("bits", [8, 4])
def test_decode_is_bit_exact(name, bits):
    got_k, got_v, ref_k, ref_v, err = run(cases()[name], bits)
    assert err == 0
    assert np.array_equal(got_k, ref_k) and np.array_equal(got_v, ref_v)


def test_v_beyond_the_fp16_range_is_saturated_and_reported():
    """V is stored as fp16: a channel whose decoded values reach 70,000 is
    saturated to 65,504 (the oracle stores the same bits) and bit 8 is set."""
    def tweak(encs):
        encs[1].offset_v[0, 3] = 70000.0
    got_k, got_v, ref_k, ref_v, err = run(cases()["ragged"], 8, layers=(0,), tweak=tweak)
    assert err == 8
    assert np.array_equal(got_k, ref_k) and np.array_equal(got_v, ref_v)
    assert (got_v == 0x7BFF).any()


def test_page_outside_the_pool_is_skipped_and_reported():
    w = cases()["ragged"]
    lay, encs = build(w, 8)
    pool = KVPool(1, lay.num_pages, w.num_kv_heads, w.head_dim, device="cuda")
    n = [lay.chunk_len[c] for c in range(len(encs))]
    tok_off = torch.tensor(np.cumsum([0] + n), dtype=torch.int32, device="cuda")
    page_off = torch.tensor(np.cumsum([0] + [len(p) for p in lay.chunk_pages]), dtype=torch.int32, device="cuda")
    pages = torch.cat(lay.chunk_pages).to(torch.int32)
    pages[0] = lay.num_pages + 3
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    cat = lambda xs: torch.from_numpy(np.ascontiguousarray(np.concatenate(xs))).cuda()
    rag_kv_decode(pool, 0, tok_off, page_off, pages.cuda(), 8, cat([e.codes_k for e in encs]),
                  cat([e.codes_v for e in encs]), cat([e.scale_k[None] for e in encs]),
                  cat([e.offset_k[None] for e in encs]), cat([e.scale_v[None] for e in encs]),
                  cat([e.offset_v[None] for e in encs]), device_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 1
