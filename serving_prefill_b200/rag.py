"""Python binding of the C ABI in include/rag_prefill.h (ctypes).

Argument marshalling only: every step of the hot path runs in the CUDA
kernels of librag.so. Tensors are torch CUDA tensors owned by the caller;
calls are asynchronous on the current torch stream unless one is passed.
There is no CPU fallback: loading fails loudly when librag.so is missing.
"""

from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_double, c_float, c_int32, c_int64, c_size_t, c_void_p

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "librag.so")

RAG_BF16, RAG_F32 = 0, 1
PAGE_SIZE = 16
KERNEL_KINDS = ("pool_write", "attn", "combine", "impact", "topk", "simt_attn", "simt_impact", "rc_plan", "rc_copy",
                "rc_gemm", "rope_table", "kv_decode", "attn_dec")

STATUS = {
    0: "ok", 1: "invalid argument", 2: "inconsistent shape", 3: "page id outside the pool",
    4: "unsupported configuration", 5: "CUDA runtime error", 6: "device pipeline wait timed out",
    7: "workspace missing or too small", 8: "chunk page count does not match its length",
    9: "a V value beyond the fp16 range was saturated",
    10: "too few free pages for the copy-on-write recompute",
}


class RagError(RuntimeError):
    def __init__(self, status: int, where: str):
        detail = ""
        if status == 5 and _lib is not None:
            detail = f", {_lib.rag_last_cuda_error().decode()}"
        super().__init__(f"{where}: {STATUS.get(status, 'unknown')} (status {status}{detail})")
        self.status = status


class RagKVPool(ctypes.Structure):
    _fields_ = [("k", c_void_p), ("v", c_void_p), ("num_layers", c_int32), ("num_pages", c_int32),
                ("num_kv_heads", c_int32), ("page_size", c_int32), ("head_dim", c_int32), ("dtype", c_int32)]


class RagBatch(ctypes.Structure):
    _fields_ = [("num_requests", c_int32), ("num_chunks", c_int32), ("num_page_refs", c_int32),
                ("total_q", c_int32), ("total_doc", c_int32), ("max_q", c_int32), ("max_doc", c_int32),
                ("max_pages", c_int32), ("req_chunk_off", c_void_p), ("chunk_doc_off", c_void_p),
                ("chunk_page_off", c_void_p), ("page_ids", c_void_p), ("q_off", c_void_p)]


_lib = None

EXPORTS = {
    "rag_abi_version": (c_int32, []),
    "rag_status_string": (ctypes.c_char_p, [c_int32]),
    "rag_num_sms": (c_int32, []),
    "rag_kv_pool_write": (c_int32, [POINTER(RagKVPool), c_int32, c_void_p, c_int32, c_int32, c_void_p, c_void_p,
                                    c_void_p, c_void_p]),
    "rag_workspace_size": (c_size_t, [POINTER(RagKVPool), POINTER(RagBatch), c_int32]),
    "rag_workspace_init": (c_int32, [c_void_p, c_size_t, c_void_p]),
    "rag_fused_prefill_attn": (c_int32, [POINTER(RagKVPool), c_int32, POINTER(RagBatch), c_void_p, c_int32,
                                         c_void_p, c_void_p, c_float, c_void_p, c_void_p, c_void_p, c_void_p,
                                         c_size_t, c_void_p]),
    "rag_fused_prefill_attn_rope": (c_int32, [POINTER(RagKVPool), c_int32, POINTER(RagBatch), c_void_p, c_int32,
                                              c_void_p, c_void_p, c_float, c_double, c_void_p, c_void_p, c_void_p,
                                              c_void_p, c_size_t, c_void_p]),
    "rag_fused_prefill_attn_static": (c_int32, [POINTER(RagKVPool), c_int32, POINTER(RagBatch), c_void_p,
                                                c_int32, c_void_p, c_void_p, c_float, c_void_p, c_void_p,
                                                c_void_p, c_void_p, c_void_p]),
    "rag_recompute_count": (c_int32, [c_int32, c_double]),
    "rag_impact_topk": (c_int32, [c_void_p, POINTER(RagBatch), c_double, c_int32, c_void_p, c_void_p, c_void_p,
                                  c_void_p]),
    "rag_last_device_error": (c_int32, [c_void_p, c_void_p, c_void_p]),
    "rag_selftest_wait_timeout": (c_int32, [c_void_p, c_int64, c_void_p]),
    "rag_kv_decode": (c_int32, [POINTER(RagKVPool), c_int32, c_int32, c_void_p, c_void_p, c_void_p, c_int32, c_int32,
                                c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "rag_recompute_plan_size": (c_size_t, [POINTER(RagBatch), c_int32]),
    "rag_recompute_plan": (c_int32, [POINTER(RagBatch), c_void_p, c_int32, c_void_p, c_void_p, c_int32, c_int32,
                                     c_void_p, c_void_p, c_size_t, c_void_p]),
    "rag_recompute_kv": (c_int32, [POINTER(RagKVPool), c_int32, POINTER(RagBatch), c_int32, c_void_p, c_size_t,
                                   c_void_p, c_int64, c_int32, c_void_p, c_void_p, c_void_p]),
    "rag_recompute_status": (c_int32, [c_void_p, c_void_p, c_void_p]),
    "rag_launch_count": (c_int64, []),
    "rag_last_cuda_error": (ctypes.c_char_p, []),
    "rag_profile_enable": (None, [c_int32]),
    "rag_profile_collect": (c_int32, [c_void_p, c_void_p, c_int32]),
    "rag_profile_peek": (c_int32, [c_void_p, c_void_p, c_int32]),
}


def lib():
    """The loaded librag.so (raises when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m serving_prefill_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in EXPORTS.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _ptr(t):
    return None if t is None else c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return c_void_p(stream.cuda_stream)


def _check(status: int, where: str):
    if status != 0:
        raise RagError(status, where)


# --------------------------------------------------------------------------- pool

class KVPool:
    """The paged pool [layers][pages][kv_heads][16][head_dim] for K and V. A
    bf16 cache keeps K in bf16 and V in fp16 (the type V enters the product
    with the attention weights in; rag_kv_pool_write and the decode and
    recompute kernels store it so)."""

    def __init__(self, num_layers, num_pages, num_kv_heads, head_dim, dtype=torch.bfloat16, device="cuda",
                 k=None, v=None):
        shape = (num_layers, num_pages, num_kv_heads, PAGE_SIZE, head_dim)
        v_dtype = torch.float16 if dtype == torch.bfloat16 else dtype
        self.k = torch.zeros(shape, dtype=dtype, device=device) if k is None else k
        self.v = torch.zeros(shape, dtype=v_dtype, device=device) if v is None else v
        assert tuple(self.k.shape) == shape and tuple(self.v.shape) == shape
        assert self.k.dtype == dtype and self.v.dtype == v_dtype
        self.c = RagKVPool(self.k.data_ptr(), self.v.data_ptr(), num_layers, num_pages, num_kv_heads, PAGE_SIZE,
                           head_dim, RAG_BF16 if dtype == torch.bfloat16 else RAG_F32)

    @property
    def num_kv_heads(self):
        return self.c.num_kv_heads


# --------------------------------------------------------------------------- batch

class Batch:
    """Batch descriptor: device int32 arrays plus host totals and maxima."""

    def __init__(self, req_chunk_off, chunk_doc_off, chunk_page_off, page_ids, q_off, device="cuda"):
        h = [torch.as_tensor(x, dtype=torch.int32).cpu() for x in
             (req_chunk_off, chunk_doc_off, chunk_page_off, page_ids, q_off)]
        self.host = h
        rc, cd, cp, pid, qo = h
        B = len(rc) - 1
        docs = [int(cd[rc[b + 1]] - cd[rc[b]]) for b in range(B)]
        pages = [int(cp[rc[b + 1]] - cp[rc[b]]) for b in range(B)]
        qs = [int(qo[b + 1] - qo[b]) for b in range(B)]
        self.dev = [t.to(device) if t.numel() > 0 else torch.zeros(1, dtype=torch.int32, device=device) for t in h]
        self.c = RagBatch(B, len(cd) - 1, len(pid), int(qo[-1]) if B else 0, int(cd[-1]) if len(cd) else 0,
                          max(qs, default=0), max(docs, default=0), max(pages, default=0),
                          *[t.data_ptr() for t in self.dev])
        self.doc_lens, self.q_lens = docs, qs

    @property
    def num_requests(self):
        return self.c.num_requests

    @property
    def total_q(self):
        return self.c.total_q

    @property
    def total_doc(self):
        return self.c.total_doc


# --------------------------------------------------------------------------- entry points

def rag_abi_version() -> int:
    return lib().rag_abi_version()


def rag_num_sms() -> int:
    return lib().rag_num_sms()


def rag_recompute_count(n_doc: int, r: float) -> int:
    return lib().rag_recompute_count(n_doc, r)


def rag_kv_pool_write(pool: KVPool, layer: int, page_ids: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                      device_err: torch.Tensor = None, stream=None):
    n_tokens = k.shape[0]
    _check(lib().rag_kv_pool_write(ctypes.byref(pool.c), layer, _ptr(page_ids), page_ids.numel(), n_tokens,
                                   _ptr(k), _ptr(v), _ptr(device_err), _stream(stream)), "rag_kv_pool_write")


def rag_workspace_size(pool: KVPool, batch: Batch, num_q_heads: int) -> int:
    n = lib().rag_workspace_size(ctypes.byref(pool.c), ctypes.byref(batch.c), num_q_heads)
    if n == 0:
        raise RagError(1, "rag_workspace_size")
    return n


def new_workspace(pool: KVPool, batch: Batch, num_q_heads: int, device="cuda", stream=None) -> torch.Tensor:
    n = rag_workspace_size(pool, batch, num_q_heads)
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    _check(lib().rag_workspace_init(_ptr(ws), n, _stream(stream)), "rag_workspace_init")
    return ws


def rag_fused_prefill_attn(pool: KVPool, layer: int, batch: Batch, q: torch.Tensor, kq: torch.Tensor,
                           vq: torch.Tensor, o: torch.Tensor, workspace: torch.Tensor, impact: torch.Tensor = None,
                           row_lse: torch.Tensor = None, sm_scale: float = 0.0, stream=None):
    num_q_heads = q.shape[1] if q.dim() == 3 else 0
    _check(lib().rag_fused_prefill_attn(ctypes.byref(pool.c), layer, ctypes.byref(batch.c), _ptr(q), num_q_heads,
                                        _ptr(kq), _ptr(vq), sm_scale, _ptr(o), _ptr(row_lse), _ptr(impact),
                                        _ptr(workspace), workspace.numel(), _stream(stream)),
           "rag_fused_prefill_attn")


def rag_fused_prefill_attn_rope(pool: KVPool, layer: int, batch: Batch, q: torch.Tensor, kq: torch.Tensor,
                                vq: torch.Tensor, o: torch.Tensor, workspace: torch.Tensor, rope_base: float,
                                impact: torch.Tensor = None, row_lse: torch.Tensor = None, sm_scale: float = 0.0,
                                stream=None):
    num_q_heads = q.shape[1] if q.dim() == 3 else 0
    _check(lib().rag_fused_prefill_attn_rope(ctypes.byref(pool.c), layer, ctypes.byref(batch.c), _ptr(q),
                                             num_q_heads, _ptr(kq), _ptr(vq), sm_scale, rope_base, _ptr(o),
                                             _ptr(row_lse), _ptr(impact), _ptr(workspace), workspace.numel(),
                                             _stream(stream)), "rag_fused_prefill_attn_rope")


def rag_fused_prefill_attn_static(pool: KVPool, layer: int, batch: Batch, q: torch.Tensor, kq: torch.Tensor,
                                  vq: torch.Tensor, o: torch.Tensor, impact: torch.Tensor = None,
                                  row_lse: torch.Tensor = None, device_err: torch.Tensor = None,
                                  sm_scale: float = 0.0, stream=None):
    """rag_fused_prefill_attn without a workspace: for callers that cannot
    allocate device memory; scratch is the library's fixed 64 MiB device array."""
    num_q_heads = q.shape[1] if q.dim() == 3 else 0
    _check(lib().rag_fused_prefill_attn_static(ctypes.byref(pool.c), layer, ctypes.byref(batch.c), _ptr(q),
                                               num_q_heads, _ptr(kq), _ptr(vq), sm_scale, _ptr(o), _ptr(row_lse),
                                               _ptr(impact), _ptr(device_err), _stream(stream)),
           "rag_fused_prefill_attn_static")


def rag_impact_topk(impact: torch.Tensor, batch: Batch, r: float, k_cap: int, topk_idx: torch.Tensor,
                    topk_val: torch.Tensor = None, k_out: torch.Tensor = None, stream=None):
    _check(lib().rag_impact_topk(_ptr(impact), ctypes.byref(batch.c), r, k_cap, _ptr(topk_idx), _ptr(topk_val),
                                 _ptr(k_out), _stream(stream)), "rag_impact_topk")


def rag_last_device_error(workspace: torch.Tensor, stream=None) -> tuple:
    bits = c_int32(0)
    st = lib().rag_last_device_error(_ptr(workspace), ctypes.byref(bits), _stream(stream))
    return st, bits.value


def rag_selftest_wait_timeout(device_err: torch.Tensor, limit_ns: int, stream=None):
    _check(lib().rag_selftest_wait_timeout(_ptr(device_err), limit_ns, _stream(stream)),
           "rag_selftest_wait_timeout")


def rag_kv_decode(pool: KVPool, layer: int, chunk_tok_off: torch.Tensor, chunk_page_off: torch.Tensor,
                  page_ids: torch.Tensor, bits: int, codes_k: torch.Tensor, codes_v: torch.Tensor,
                  scale_k: torch.Tensor, offset_k: torch.Tensor, scale_v: torch.Tensor, offset_v: torch.Tensor,
                  device_err: torch.Tensor = None, stream=None):
    _check(lib().rag_kv_decode(ctypes.byref(pool.c), layer, chunk_tok_off.numel() - 1, _ptr(chunk_tok_off),
                               _ptr(chunk_page_off), _ptr(page_ids), page_ids.numel(), bits, _ptr(codes_k),
                               _ptr(codes_v), _ptr(scale_k), _ptr(offset_k), _ptr(scale_v), _ptr(offset_v),
                               _ptr(device_err), _stream(stream)), "rag_kv_decode")


def rag_recompute_plan_size(batch: Batch, k_cap: int) -> int:
    n = lib().rag_recompute_plan_size(ctypes.byref(batch.c), k_cap)
    if n == 0:
        raise RagError(1, "rag_recompute_plan_size")
    return n


def rag_recompute_plan(batch: Batch, topk_idx: torch.Tensor, k_cap: int, k: torch.Tensor, free_pages: torch.Tensor,
                       page_ids_out: torch.Tensor, plan: torch.Tensor, x_by_selection: bool = False, stream=None):
    _check(lib().rag_recompute_plan(ctypes.byref(batch.c), _ptr(topk_idx), k_cap, _ptr(k), _ptr(free_pages),
                                    free_pages.numel(), 1 if x_by_selection else 0, _ptr(page_ids_out), _ptr(plan),
                                    plan.numel() * plan.element_size(), _stream(stream)), "rag_recompute_plan")


def rag_recompute_kv(pool: KVPool, layer: int, batch: Batch, k_cap: int, plan: torch.Tensor, x: torch.Tensor,
                     w_k: torch.Tensor, w_v: torch.Tensor, stream=None):
    _check(lib().rag_recompute_kv(ctypes.byref(pool.c), layer, ctypes.byref(batch.c), k_cap, _ptr(plan),
                                  plan.numel() * plan.element_size(), _ptr(x), x.shape[0], x.shape[1], _ptr(w_k),
                                  _ptr(w_v), _stream(stream)), "rag_recompute_kv")


def rag_recompute_status(plan: torch.Tensor, stream=None) -> tuple:
    counts = (c_int32 * 3)()
    st = lib().rag_recompute_status(_ptr(plan), ctypes.cast(counts, c_void_p), _stream(stream))
    return st, (counts[0], counts[1], counts[2])


def rag_launch_count() -> int:
    return lib().rag_launch_count()


def rag_profile_enable(on: bool):
    lib().rag_profile_enable(1 if on else 0)


def rag_profile_peek() -> dict:
    n = len(KERNEL_KINDS)
    ms = (c_double * n)()
    cnt = (c_int64 * n)()
    _check(lib().rag_profile_peek(ctypes.cast(ms, c_void_p), ctypes.cast(cnt, c_void_p), n), "rag_profile_peek")
    return {k: (ms[i], cnt[i]) for i, k in enumerate(KERNEL_KINDS)}


def rag_profile_collect() -> dict:
    n = len(KERNEL_KINDS)
    ms = (c_double * n)()
    cnt = (c_int64 * n)()
    _check(lib().rag_profile_collect(ctypes.cast(ms, c_void_p), ctypes.cast(cnt, c_void_p), n),
           "rag_profile_collect")
    return {k: (ms[i], cnt[i]) for i, k in enumerate(KERNEL_KINDS)}


def topk_capacity(batch: Batch, r: float) -> int:
    """Row length for the top-k outputs: k of the request with the most doc tokens."""
    return max(1, rag_recompute_count(max(batch.doc_lens, default=0), r))
