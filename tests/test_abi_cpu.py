"""The C ABI without a GPU: the library loads, exports every entry point the
header declares, and rejects bad arguments before launching anything."""

import ctypes
import os
import re
import subprocess

import pytest
import torch

import oracle.prefill as orc
import serving_prefill_b200 as sp
from serving_prefill_b200.rag import RagBatch, RagKVPool, lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rag_prefill.h")


def declared_entry_points():
    text = open(HEADER).read()
    return re.findall(r"RAG_API\s+[\w\s\*]+?\b(rag_\w+)\s*\(", text)


def test_header_declares_entry_points():
    names = declared_entry_points()
    for must in ("rag_kv_pool_write", "rag_fused_prefill_attn", "rag_impact_topk", "rag_workspace_size",
                 "rag_last_device_error", "rag_recompute_count"):
        assert must in names


def test_library_exports_every_declared_symbol():
    handle = lib()
    out = subprocess.run(["nm", "-D", "--defined-only", sp.rag.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\sT\s(\w+)", out))
    for name in declared_entry_points():
        assert name in exported, name
        assert getattr(handle, name) is not None
    # internal symbols stay hidden
    assert not any(s.startswith("_ZN3rag") for s in exported)


def test_abi_version():
    assert sp.rag_abi_version() == 1


def test_recompute_count_matches_oracle():
    for r in (0.05, 0.1, 0.15, 0.3):
        for n in list(range(1, 3000)) + [10000, 65536, 100003]:
            assert sp.rag_recompute_count(n, r) == orc.recompute_count(n, r)
    assert sp.rag_recompute_count(0, 0.1) == 0


def fake_pool(head_dim=128, dtype=0, layers=1, pages=64, heads=8, page_size=16):
    return RagKVPool(0x10000, 0x20000, layers, pages, heads, page_size, head_dim, dtype)


def fake_batch(B=2, q=(10, 20), docs=(100, 50)):
    pages = [-(-d // 16) for d in docs]
    return RagBatch(B, B, sum(pages), sum(q), sum(docs), max(q), max(docs), max(pages),
                    0x30000, 0x31000, 0x32000, 0x33000, 0x34000)


def attn(pool, batch, hq=32, q=0x40000, kq=0x50000, vq=0x60000, o=0x70000, ws=0x80000, ws_bytes=1 << 30,
         lse=None, impact=None):
    return lib().rag_fused_prefill_attn(ctypes.byref(pool), 0, ctypes.byref(batch), q, hq, kq, vq, 0.0, o, lse,
                                        impact, ws, ws_bytes, None)


def test_validation_rejects_before_launch():
    L = lib()
    assert L.rag_fused_prefill_attn(None, 0, None, None, 32, None, None, 0.0, None, None, None, None, 0, None) == 1
    pool, batch = fake_pool(), fake_batch()
    assert attn(fake_pool(page_size=32), batch) == 4           # page size
    assert attn(fake_pool(head_dim=64), batch) == 4            # bf16 needs head_dim 128
    assert attn(fake_pool(dtype=7), batch) == 4                # unknown dtype
    assert attn(pool, batch, hq=30) == 2                       # H_q not a multiple of H_kv
    assert attn(pool, batch, q=0x40001) == 1                   # misaligned Q
    assert attn(pool, batch, ws=0x80010) == 7                  # workspace alignment
    assert attn(pool, batch, ws_bytes=1024) == 7               # workspace too small
    assert attn(pool, batch, hq=8 * 256, ws_bytes=1 << 40) == 4  # group of 256 does not divide 128 rows
    big = fake_pool(layers=4096, pages=4096, heads=16)         # 2^32 pool rows
    assert attn(big, batch) == 4
    bad = fake_batch()
    bad.max_q = 1000                                           # max above total
    assert attn(pool, bad) == 2
    many = fake_batch()
    many.num_requests = 4097                                   # above the 4,096 requests a batch may hold
    assert attn(pool, many) == 4


def test_pool_write_validation():
    L = lib()
    pool = fake_pool()
    assert L.rag_kv_pool_write(ctypes.byref(pool), 5, 0x1000, 3, 40, 0x2000, 0x3000, None, None) == 1  # layer
    assert L.rag_kv_pool_write(ctypes.byref(pool), 0, 0x1000, 2, 40, 0x2000, 0x3000, None, None) == 2  # pages
    assert L.rag_kv_pool_write(ctypes.byref(pool), 0, 0x1000, 3, 40, 0x2001, 0x3000, None, None) == 1  # align
    assert L.rag_kv_pool_write(ctypes.byref(pool), 0, 0x1000, 0, 0, 0x2000, 0x3000, None, None) == 0   # empty


def test_topk_validation():
    L = lib()
    batch = fake_batch()
    assert L.rag_impact_topk(0x1000, ctypes.byref(batch), 0.0, 100, 0x2000, None, None, None) == 1
    assert L.rag_impact_topk(0x1000, ctypes.byref(batch), 1.0, 100, 0x2000, None, None, None) == 1
    assert L.rag_impact_topk(0x1000, ctypes.byref(batch), 0.1, 5, 0x2000, None, None, None) == 2   # k_cap < 10
    assert L.rag_impact_topk(None, ctypes.byref(batch), 0.1, 10, 0x2000, None, None, None) == 1
    huge = fake_batch(docs=(100000, 50))
    assert L.rag_impact_topk(0x1000, ctypes.byref(huge), 0.5, 60000, 0x2000, None, None, None) == 4


def test_workspace_size_grows_with_batch():
    pool = fake_pool()
    small = lib().rag_workspace_size(ctypes.byref(pool), ctypes.byref(fake_batch()), 32)
    large = lib().rag_workspace_size(ctypes.byref(pool), ctypes.byref(fake_batch(q=(100, 200), docs=(4000, 900))), 32)
    assert 0 < small < large
    assert lib().rag_workspace_size(ctypes.byref(pool), ctypes.byref(fake_batch()), 30) == 0


def test_status_strings():
    for s in range(10):
        assert lib().rag_status_string(s).decode() != "unknown status"
    assert lib().rag_status_string(99).decode() == "unknown status"


def test_binding_batch_marshalling_on_cpu():
    from workloads import get_workload, make_layout
    lay = make_layout(get_workload("batched16"))
    b = sp.Batch(lay.req_chunk_off, lay.chunk_doc_off, lay.chunk_page_off, lay.page_ids, lay.q_off, device="cpu")
    assert b.num_requests == 16 and b.total_q == lay.total_q and b.total_doc == lay.total_doc
    assert b.c.max_doc == max(lay.doc_lens) and b.c.max_q == max(lay.q_lens)
    assert b.c.max_pages == max(lay.page_counts)
    assert sp.topk_capacity(b, 0.1) == orc.recompute_count(max(lay.doc_lens), 0.1)


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    import serving_prefill_b200.rag as rag
    monkeypatch.setattr(rag, "_lib", None)
    monkeypatch.setattr(rag, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        rag.lib()


def test_last_cuda_error_names_a_cuda_error():
    name = lib().rag_last_cuda_error().decode()
    assert name.startswith("cuda")
