"""Plain fp64 definition of the precomputed-KV RAG prefill hot path.

TEST INFRASTRUCTURE: only the tests, the smoke check and the benchmark's
CPU-baseline leg use this module. It shares no code with the CUDA library and
imports nothing from it.

What it computes, step by step, in the pages' order:

1. Pool write (TurboRAG page, "Technical Details", KV precompute equation
   K_l^(j) = W_K^l Encode(D_j), and the `precompute_kv_cache` listing): a
   chunk's per-layer K, V [n, H_kv, d] are stored in fixed 16-token pages of a
   pool [layers][pages][H_kv][16][d]. The page layout is this library's choice
   (the TurboRAG page's related-work section points at PagedAttention); each
   chunk starts on a fresh page and the unused tail slots of its last page are
   zero. The storage format is this library's choice too (the pages fix no
   precision): in a bf16 cache, K is stored as bf16 and V as the fp16 value of
   its bf16 value (round to nearest even; magnitudes beyond 65504 saturate),
   the operand type in which V enters the product with the normalised
   weights. Every bf16 value of magnitude in [2^-14, 65280] is exact in fp16;
   smaller ones move by less than 2^-25. The query block's own V_q enters the
   product in the same form.
2. Concat (TurboRAG page, "Technical Details", K_combined = Concat(K^(1), ...,
   K^(m), K^(Q)); CacheBlend page, "Mathematical formulation",
   K_concat = [K_1; ...; K_m; K_q]): the request's chunks in retrieval order
   along the sequence axis, then the query block's own K_q, V_q.
3. Attention (TurboRAG page, "Causal vs non-causal attention",
   softmax(Q K^T / sqrt(d_k) + M_causal) V): query token j of a request sits at
   logical position N_doc + j and sees every key i <= N_doc + j; all doc keys
   are visible to every query token, and the mask is causal only inside the
   query block. Query head h reads KV head floor(h / G), G = H_q / H_kv.
4. Impact (CacheBlend page, "Mathematical formulation", Impact(i) = sum over
   j outside doc(i) of alpha_{j,i}; and the `select_tokens_for_recompute`
   listing, which sums the softmax weights of the query rows over each column):
   alpha are the normalised weights of step 3; the sum runs over the query
   tokens (which belong to no document) and is averaged over the H_q query
   heads, so the impacts of all N_doc + q columns add up to q.
5. Recompute count and top-k (CacheBlend page, "Recompute ratio trade-off",
   count = r * sum |D_i|; listing: max(1, int(doc_token_count * ratio)) and
   torch.topk over the doc slice): the k doc positions of largest impact,
   ordered by (impact descending, position ascending).

All arithmetic is fp64 on the exact values of the bf16/fp32 inputs.
Parity pins for every step live in tests/test_oracle_*.py.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

PAGE_SIZE = 16


# --------------------------------------------------------------------------
# storage helpers: raw bits of the storage dtype <-> exact fp64 values
# --------------------------------------------------------------------------

def to_bits(t: torch.Tensor) -> np.ndarray:
    """Raw storage bits of a bf16 (uint16) or fp32 (uint32) tensor."""
    t = t.contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16).copy()
    if t.dtype == torch.float32:
        return t.view(torch.int32).numpy().view(np.uint32).copy()
    raise TypeError(f"unsupported storage dtype {t.dtype}")


def bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Exact fp64 value of stored bits (bf16 is the top half of an fp32)."""
    if b.dtype == np.uint16:
        return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if b.dtype == np.uint32:
        return b.view(np.float32).astype(np.float64)
    raise TypeError(f"unsupported bits dtype {b.dtype}")


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()


F16_MAX = 65504.0


def f16_bits_sat(x: np.ndarray) -> np.ndarray:
    """fp64 values -> fp16 bits, rounded once to nearest (ties to even),
    magnitudes beyond 65504 (inf included) saturated to +-65504, nan kept."""
    x = np.asarray(x, dtype=np.float64)
    x = np.where(np.isnan(x), x, np.clip(x, -F16_MAX, F16_MAX))
    return x.astype(np.float16).view(np.uint16)


def v_operand_bits(b: np.ndarray) -> np.ndarray:
    """Stored V of a bf16 cache: bf16 bits -> fp16 bits of the same value
    (f16_bits_sat of the exact bf16 value)."""
    return f16_bits_sat(bits_to_f64(b))


def f16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Exact fp64 value of fp16 bits."""
    return np.asarray(b, dtype=np.uint16).view(np.float16).astype(np.float64)


# --------------------------------------------------------------------------
# step 1: pool write
# --------------------------------------------------------------------------

def new_pool(num_layers: int, num_pages: int, num_kv_heads: int, head_dim: int,
             bits_dtype) -> np.ndarray:
    return np.zeros((num_layers, num_pages, num_kv_heads, PAGE_SIZE, head_dim), dtype=bits_dtype)


def pool_write(pool: np.ndarray, layer: int, page_ids, chunk_bits: np.ndarray) -> None:
    """Store one chunk's dense [n, H_kv, d] values (raw bits) into its pages.

    Token t of the chunk goes to page page_ids[t // 16], slot t % 16. The
    slots of the last page past the chunk's end are zeroed.
    """
    n = chunk_bits.shape[0]
    page_ids = np.asarray(page_ids, dtype=np.int64)
    assert len(page_ids) == -(-n // PAGE_SIZE), "one page per 16 tokens"
    for t in range(n):
        pool[layer, page_ids[t // PAGE_SIZE], :, t % PAGE_SIZE, :] = chunk_bits[t]
    for t in range(n, len(page_ids) * PAGE_SIZE):
        pool[layer, page_ids[t // PAGE_SIZE], :, t % PAGE_SIZE, :] = 0


# --------------------------------------------------------------------------
# step 2: Concat through the page table
# --------------------------------------------------------------------------

def gather(pool: np.ndarray, layer: int, chunks) -> np.ndarray:
    """[K_1; ...; K_m] for one request, as raw bits [N_doc, H_kv, d].

    `chunks` lists (page_ids, n_tokens) per chunk in retrieval order.
    """
    parts = []
    for page_ids, n in chunks:
        page_ids = np.asarray(page_ids, dtype=np.int64)
        t = np.arange(n)
        parts.append(pool[layer, page_ids[t // PAGE_SIZE], :, t % PAGE_SIZE, :])
    if not parts:
        return pool[layer, :0, :, 0, :]
    return np.concatenate(parts, axis=0)


# --------------------------------------------------------------------------
# step 2b (optional): RoPE position re-basing of the cached keys
# --------------------------------------------------------------------------
#
# TurboRAG page, "Implementation": with rotary position embeddings, the
# position ids used when a chunk's cache is precomputed and those used at
# inference must agree. A chunk precomputed on its own carries RoPE at its
# local positions 0 .. n_c - 1; in the concatenated sequence it starts at
# offset o (the doc tokens of the chunks before it). Re-basing rotates every
# cached key by the angle o * theta_i of its rotary pair, which moves it to
# position o + t (rotations of one pair add their angles). Convention (Llama's
# rotary embedding): pair i couples channels i and i + d/2, theta_i =
# base^(-2 i / d). The re-based key is held in the cache dtype: the rotation
# is exact (fp64) and the result is rounded once to bf16.

def rope_theta_i(head_dim: int, base: float) -> np.ndarray:
    """Angle per position of each rotary pair: base^(-2 i / d), i < d / 2."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * i / head_dim)


def rope_rotate(k: np.ndarray, offset: int, base: float) -> np.ndarray:
    """Rotate keys [..., d] (fp64) by offset positions: pair (i, i + d/2) turns
    by offset * theta_i."""
    d = k.shape[-1]
    ang = float(offset) * rope_theta_i(d, base)
    c, s = np.cos(ang), np.sin(ang)
    a, b = k[..., : d // 2], k[..., d // 2:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def rope_rebase_bits(k_bits: np.ndarray, offset: int, base: float) -> np.ndarray:
    """Re-based cached keys in the cache dtype (bf16 bits), rounded once."""
    r = rope_rotate(bits_to_f64(k_bits), offset, base)
    t = torch.from_numpy(np.ascontiguousarray(r)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def gather_rebased(pool: np.ndarray, layer: int, chunks, base: float) -> np.ndarray:
    """gather() with every chunk's keys re-based to its offset in the request."""
    parts, at = [], 0
    for page_ids, n in chunks:
        part = gather(pool, layer, [(page_ids, n)])
        parts.append(rope_rebase_bits(part, at, base))
        at += n
    if not parts:
        return pool[layer, :0, :, 0, :]
    return np.concatenate(parts, axis=0)


# --------------------------------------------------------------------------
# step 3 + 4: masked softmax attention and Impact for one request
# --------------------------------------------------------------------------

def kv_head_of(h: int, group: int) -> int:
    """Query head h reads KV head h // G (consecutive query heads share one)."""
    return h // group


def visible(i, j, n_doc):
    """Key position i is visible to query token j (at position n_doc + j)."""
    return i <= n_doc + j


def attend_request(q: np.ndarray, kcat: np.ndarray, vcat: np.ndarray, n_doc: int,
                   scale: float, want_impact: bool = True, want_alpha: bool = False):
    """Attention of one request's query block over [K_1; ...; K_m; K_q].

    q: [q_len, H_q, d]; kcat, vcat: [n_doc + q_len, H_kv, d] (fp64).
    Returns O [q_len, H_q, d], m [q_len, H_q] (max scaled score per row),
    l [q_len, H_q] (sum of exp(s - m) per row), impact [n_doc + q_len] or None,
    and alpha [H_q, q_len, n_doc + q_len] when asked for.
    """
    q_len, hq, d = q.shape
    n_tot, hk, _ = kcat.shape
    assert n_tot == n_doc + q_len
    group = hq // hk
    o = np.zeros((q_len, hq, d))
    m = np.zeros((q_len, hq))
    l = np.zeros((q_len, hq))
    impact = np.zeros(n_tot) if want_impact else None
    alpha_all = np.zeros((hq, q_len, n_tot)) if want_alpha else None
    vis = visible(np.arange(n_tot)[None, :], np.arange(q_len)[:, None], n_doc)
    for h in range(hq):
        g = kv_head_of(h, group)
        s = scale * (q[:, h, :] @ kcat[:, g, :].T)          # [q_len, n_tot]
        s = np.where(vis, s, -np.inf)
        m_h = s.max(axis=1)
        p = np.exp(s - m_h[:, None])
        l_h = p.sum(axis=1)
        alpha = p / l_h[:, None]
        o[:, h, :] = alpha @ vcat[:, g, :]
        m[:, h] = m_h
        l[:, h] = l_h
        if want_impact:
            impact += alpha.sum(axis=0) / hq
        if want_alpha:
            alpha_all[h] = alpha
    return o, m, l, impact, alpha_all


# --------------------------------------------------------------------------
# step 5: recompute count and top-k
# --------------------------------------------------------------------------

def recompute_count(n_doc: int, r: float) -> int:
    """k = max(1, int(N_doc * r)), with the product taken in double precision.

    A request with no doc tokens has nothing to select: k = 0 (the listing's
    max(1, .) is read as applying to a non-empty doc slice).
    """
    if n_doc <= 0:
        return 0
    return max(1, int(n_doc * r))


def select_topk(impact_doc: np.ndarray, k: int) -> np.ndarray:
    """Positions of the k largest impacts, by (impact desc, position asc)."""
    n = len(impact_doc)
    order = np.lexsort((np.arange(n), -np.asarray(impact_doc, dtype=np.float64)))
    return order[:k].astype(np.int64)


# --------------------------------------------------------------------------
# whole-batch driver over the seeded workloads
# --------------------------------------------------------------------------

@dataclass
class OracleResult:
    o: np.ndarray                      # [total_q, H_q, d]
    m: np.ndarray                      # [total_q, H_q]
    l: np.ndarray                      # [total_q, H_q]
    impact: np.ndarray = None          # concatenated per-request [N_doc_b + q_b] segments
    k: list = field(default_factory=list)
    topk: list = field(default_factory=list)   # per request: int64 positions
    pool_k: np.ndarray = None          # raw bits [1, pages, H_kv, 16, d] of this layer
    pool_v: np.ndarray = None          # (V of a bf16 cache: fp16 bits)


def build_layer_pool(lay, inputs, bits_dtype):
    w = lay.workload
    pk = new_pool(1, lay.num_pages, w.num_kv_heads, w.head_dim, bits_dtype)
    pv = new_pool(1, lay.num_pages, w.num_kv_heads, w.head_dim, bits_dtype)
    for c, pages in enumerate(lay.chunk_pages):
        vb = to_bits(inputs.chunk_v[c])
        pool_write(pk, 0, pages.numpy(), to_bits(inputs.chunk_k[c]))
        pool_write(pv, 0, pages.numpy(), v_operand_bits(vb) if bits_dtype == np.uint16 else vb)
    return pk, pv


def v_values(bits: np.ndarray) -> np.ndarray:
    """Exact values of stored V bits: fp16 in a bf16 cache, fp32 in an fp32 one."""
    return f16_bits_to_f64(bits) if bits.dtype == np.uint16 else bits_to_f64(bits)


def run_workload_layer(lay, inputs, want_impact: bool, scale: float = None,
                       keep_pool: bool = False, rope_base: float = None) -> OracleResult:
    """Oracle for one layer of a generated batch (all requests). rope_base:
    re-base the cached keys to their concatenated positions (None: as stored)."""
    w = lay.workload
    d = w.head_dim
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    bits_dtype = np.uint16 if w.dtype == "bf16" else np.uint32
    pk, pv = build_layer_pool(lay, inputs, bits_dtype)
    q_all = to_f64(inputs.q)
    kq_all = to_f64(inputs.kq)
    vq_bits = to_bits(inputs.vq)
    vq_all = v_values(v_operand_bits(vq_bits) if bits_dtype == np.uint16 else vq_bits)
    tq = lay.total_q
    o = np.zeros((tq, w.num_q_heads, d))
    m = np.zeros((tq, w.num_q_heads))
    l = np.zeros((tq, w.num_q_heads))
    impacts, ks, tops = [], [], []
    q0 = 0
    for b, cs in enumerate(lay.req_chunks):
        ql = lay.q_lens[b]
        chunks = [(lay.chunk_pages[c].numpy(), lay.chunk_len[c]) for c in cs]
        if rope_base is None:
            kd = bits_to_f64(gather(pk, 0, chunks))
        else:
            if bits_dtype != np.uint16:
                raise TypeError("re-basing is defined for bf16 caches")
            kd = bits_to_f64(gather_rebased(pk, 0, chunks, rope_base))
        vd = v_values(gather(pv, 0, chunks))
        n_doc = kd.shape[0]
        kcat = np.concatenate([kd, kq_all[q0:q0 + ql]], axis=0)
        vcat = np.concatenate([vd, vq_all[q0:q0 + ql]], axis=0)
        ob, mb, lb, ib, _ = attend_request(q_all[q0:q0 + ql], kcat, vcat, n_doc, scale,
                                           want_impact=want_impact)
        o[q0:q0 + ql], m[q0:q0 + ql], l[q0:q0 + ql] = ob, mb, lb
        if want_impact:
            impacts.append(ib)
            k = recompute_count(n_doc, w.r)
            ks.append(k)
            tops.append(select_topk(ib[:n_doc], k))
        q0 += ql
    res = OracleResult(o=o, m=m, l=l)
    if want_impact:
        res.impact = np.concatenate(impacts) if impacts else np.zeros(0)
        res.k, res.topk = ks, tops
    if keep_pool:
        res.pool_k, res.pool_v = pk, pv
    return res


def run_workload(lay, layer_inputs_fn, layers=None) -> dict:
    """Oracle for every requested layer; impact and top-k on the impact layer."""
    w = lay.workload
    layers = range(w.num_layers) if layers is None else layers
    out = {}
    for layer in layers:
        out[layer] = run_workload_layer(lay, layer_inputs_fn(layer),
                                        want_impact=(layer == w.impact_layer_index))
    return out
