"""Workload recipes and seeded generators.

Shapes follow the pages' RAG setting: a handful of retrieved document chunks of
hundreds to thousands of tokens (TurboRAG, "Technical Details / KV cache
precompute"; CacheBlend, "Experimental results", 4-document RAG), a query of
about a hundred tokens (TurboRAG, "Complexity analysis", 10,000 doc + 100 query
tokens) and a recompute ratio r in 0.05-0.15 (CacheBlend, "Recompute ratio").
The pages' QA datasets and model weights are not available; these seeded
draws stand in for the per-chunk KV a model would have produced.

Distribution of the synthetic KV ("lognormal"): every value is N(0, 1) times a
per-channel scale; the scales are drawn lognormal(0, 0.5) per (layer, KV head,
channel), separately for K and for V, and `n_outliers` channels per
(layer, KV head) get their scale multiplied by `outlier_gain`. The same scales
apply to every chunk and to the query's own K/V of that layer. Q is N(0, 1).
Values are drawn in fp32 and rounded once to the storage dtype; both the CUDA
path and the oracle read the rounded values.
"""

from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field

import torch

PAGE_SIZE = 16


@dataclass(frozen=True)
class Workload:
    name: str
    num_layers: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    dtype: str                      # "bf16" or "f32"
    r: float                        # recompute ratio
    seed: int
    kv_dist: str = "lognormal"      # "normal" or "lognormal"
    n_outliers: int = 2
    outlier_gain: float = 8.0
    impact_layer: int = -1          # -1: the last layer
    # one request with fixed chunks ("fixed") or requests drawn from a shared
    # pool of precomputed chunks ("pooled")
    kind: str = "fixed"
    chunk_lens: tuple = ()
    q_len: int = 0
    n_requests: int = 0
    n_pool_chunks: int = 0
    chunk_len_range: tuple = (0, 0)
    chunks_per_req: tuple = (0, 0)
    q_range: tuple = (0, 0)
    # decode steps: every request also holds a private chunk (its prompt and the
    # tokens generated so far) of a length drawn from this range, after its
    # retrieved chunks; the query block is the one new token
    context_range: tuple = (0, 0)
    select: bool = True             # run Impact and the top-k (prefill) or not (decode)
    d_model: int = 4096             # hidden size feeding the K/V projections (selective recompute)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def elem_bytes(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    @property
    def impact_layer_index(self):
        """The layer whose attention feeds Impact and the top-k; None for decode."""
        if not self.select:
            return None
        return self.num_layers - 1 if self.impact_layer < 0 else self.impact_layer


WORKLOADS = {
    # 1 layer, 2 query heads sharing 1 KV head, d 64, fp32, 32/48/40 + 8 query
    "tiny": Workload(
        name="tiny", num_layers=1, num_q_heads=2, num_kv_heads=1, head_dim=64,
        dtype="f32", r=0.1, seed=1000, kv_dist="normal", n_outliers=0,
        chunk_lens=(32, 48, 40), q_len=8),
    # Llama-2-7B-shaped single layer, MHA 32 heads, 4 x 512 + 64 query
    "llama2_7b_l1": Workload(
        name="llama2_7b_l1", num_layers=1, num_q_heads=32, num_kv_heads=32,
        head_dim=128, dtype="bf16", r=0.1, seed=1001,
        chunk_lens=(512,) * 4, q_len=64),
    # Llama-3-8B-shaped, 32 layers, 32q/8kv, 10 x 1000 + 100 query
    "llama3_8b_l32": Workload(
        name="llama3_8b_l32", num_layers=32, num_q_heads=32, num_kv_heads=8,
        head_dim=128, dtype="bf16", r=0.15, seed=1002,
        chunk_lens=(1000,) * 10, q_len=100),
    # 16 requests, 4-8 chunks each drawn with replacement from 256 chunks
    "batched16": Workload(
        name="batched16", num_layers=1, num_q_heads=32, num_kv_heads=8,
        head_dim=128, dtype="bf16", r=0.1, seed=1003, kind="pooled",
        n_requests=16, n_pool_chunks=256, chunk_len_range=(256, 1024),
        chunks_per_req=(4, 8), q_range=(32, 128)),
    # decode over the fused cache: the batched16 requests one generation step
    # later; each holds its prompt (32-128 tokens) and up to 256 generated
    # tokens as a private chunk and attends with one new token
    "decode16": Workload(
        name="decode16", num_layers=1, num_q_heads=32, num_kv_heads=8,
        head_dim=128, dtype="bf16", r=0.1, seed=1005, kind="pooled",
        n_requests=16, n_pool_chunks=256, chunk_len_range=(256, 1024),
        chunks_per_req=(4, 8), q_range=(1, 1), context_range=(33, 384), select=False),
    # 70B-shaped single layer, 64q/8kv, 32 x 2048 + 256 query, 4 outliers
    "long70b": Workload(
        name="long70b", num_layers=1, num_q_heads=64, num_kv_heads=8,
        head_dim=128, dtype="bf16", r=0.05, seed=1004, n_outliers=4,
        chunk_lens=(2048,) * 32, q_len=256, d_model=8192),
}

# index order of the workloads as the headline configuration list gives them
WORKLOAD_ORDER = ["tiny", "llama2_7b_l1", "llama3_8b_l32", "batched16", "long70b"]


def get_workload(name_or_index) -> Workload:
    if isinstance(name_or_index, int) or str(name_or_index).isdigit():
        return WORKLOADS[WORKLOAD_ORDER[int(name_or_index)]]
    return WORKLOADS[name_or_index]


def scaled(w: Workload, **overrides) -> Workload:
    """A copy of a workload with some fields replaced (smaller test cases)."""
    name = overrides.pop("name", w.name + "_scaled")
    return dataclasses.replace(w, name=name, **overrides)


def _gen(seed: int, *tags: int) -> torch.Generator:
    """An independent CPU generator for one sub-stream of a workload seed."""
    s = seed
    for t in tags:
        s = (s * 1_000_003 + 7919 * (t + 1)) % (2**63 - 1)
    g = torch.Generator(device="cpu")
    g.manual_seed(s)
    return g


# sub-stream tags
_T_LAYOUT, _T_SCALE, _T_Q, _T_K, _T_V, _T_KQ, _T_VQ, _T_X, _T_WK, _T_WV, _T_CODES = range(11)


@dataclass
class BatchLayout:
    """Which chunks each request retrieves and where their pages live.

    Distinct chunks are the precomputed units held in the pool (`chunk_len`,
    `chunk_pages`). A request lists distinct chunks in retrieval order; the
    same chunk may appear in several requests or twice in one (pooled draws).
    The flat int32 arrays are the batch descriptor the kernels take:
      req_chunk_off  [B+1]  request b owns chunk-list entries [off[b], off[b+1])
      chunk_doc_off  [C+1]  cumulative doc tokens over the chunk list
      chunk_page_off [C+1]  cumulative pages over the chunk list
      page_ids       [P]    physical page of each referenced page, in order
      q_off          [B+1]  cumulative query tokens
    """
    workload: Workload
    num_pages: int
    chunk_len: list                     # per distinct chunk
    chunk_pages: list                   # per distinct chunk: LongTensor of page ids
    req_chunks: list                    # per request: list of distinct chunk ids
    q_lens: list                        # per request
    req_chunk_off: torch.Tensor = field(default=None)
    chunk_doc_off: torch.Tensor = field(default=None)
    chunk_page_off: torch.Tensor = field(default=None)
    page_ids: torch.Tensor = field(default=None)
    q_off: torch.Tensor = field(default=None)

    @property
    def num_requests(self) -> int:
        return len(self.req_chunks)

    @property
    def doc_lens(self) -> list:
        return [sum(self.chunk_len[c] for c in cs) for cs in self.req_chunks]

    @property
    def page_counts(self) -> list:
        return [sum(len(self.chunk_pages[c]) for c in cs) for cs in self.req_chunks]

    @property
    def total_q(self) -> int:
        return sum(self.q_lens)

    @property
    def total_doc(self) -> int:
        return sum(self.doc_lens)

    def with_page_permutation(self, seed: int) -> "BatchLayout":
        """Same logical content, every page moved to another physical slot."""
        g = _gen(seed, 99)
        perm = torch.randperm(self.num_pages, generator=g)
        pages = [perm[p] for p in self.chunk_pages]
        out = dataclasses.replace(self, chunk_pages=pages)
        _flatten(out)
        return out

    def with_chunk_order(self, orders: list) -> "BatchLayout":
        """Same chunks per request, retrieved in another order."""
        req = [[cs[i] for i in order] for cs, order in zip(self.req_chunks, orders)]
        out = dataclasses.replace(self, req_chunks=req)
        _flatten(out)
        return out


def _flatten(lay: BatchLayout) -> None:
    rc, cd, cp, pid, qo = [0], [0], [0], [], [0]
    for cs, q in zip(lay.req_chunks, lay.q_lens):
        for c in cs:
            cd.append(cd[-1] + lay.chunk_len[c])
            cp.append(cp[-1] + len(lay.chunk_pages[c]))
            pid.extend(int(p) for p in lay.chunk_pages[c])
        rc.append(rc[-1] + len(cs))
        qo.append(qo[-1] + q)
    i32 = torch.int32
    lay.req_chunk_off = torch.tensor(rc, dtype=i32)
    lay.chunk_doc_off = torch.tensor(cd, dtype=i32)
    lay.chunk_page_off = torch.tensor(cp, dtype=i32)
    lay.page_ids = torch.tensor(pid, dtype=i32)
    lay.q_off = torch.tensor(qo, dtype=i32)


def make_layout(w: Workload) -> BatchLayout:
    g = _gen(w.seed, _T_LAYOUT)
    if w.kind == "fixed":
        chunk_len = list(w.chunk_lens)
        req_chunks = [list(range(len(chunk_len)))]
        q_lens = [w.q_len]
    else:
        lo, hi = w.chunk_len_range
        chunk_len = torch.randint(lo, hi + 1, (w.n_pool_chunks,), generator=g).tolist()
        req_chunks, q_lens = [], []
        for _ in range(w.n_requests):
            n = int(torch.randint(w.chunks_per_req[0], w.chunks_per_req[1] + 1, (1,), generator=g))
            req_chunks.append(torch.randint(0, w.n_pool_chunks, (n,), generator=g).tolist())
            q_lens.append(int(torch.randint(w.q_range[0], w.q_range[1] + 1, (1,), generator=g)))
        if w.context_range[1] > 0:
            for cs in req_chunks:
                cs.append(len(chunk_len))
                chunk_len.append(int(torch.randint(w.context_range[0], w.context_range[1] + 1, (1,), generator=g)))
    n_pages = [-(-n // PAGE_SIZE) for n in chunk_len]
    num_pages = sum(n_pages)
    perm = torch.randperm(num_pages, generator=g)
    chunk_pages, at = [], 0
    for n in n_pages:
        chunk_pages.append(perm[at:at + n].clone())
        at += n
    lay = BatchLayout(workload=w, num_pages=num_pages, chunk_len=chunk_len,
                      chunk_pages=chunk_pages, req_chunks=req_chunks, q_lens=q_lens)
    _flatten(lay)
    return lay


@dataclass
class LayerInputs:
    """One layer's values: per distinct chunk K/V, and the batch's Q, K_q, V_q."""
    chunk_k: list          # per distinct chunk: [len, H_kv, d] (storage dtype)
    chunk_v: list
    q: torch.Tensor        # [total_q, H_q, d]
    kq: torch.Tensor       # [total_q, H_kv, d]
    vq: torch.Tensor


def _scales(w: Workload, layer: int, which: int) -> torch.Tensor:
    """Per (KV head, channel) scale for K (which=0) or V (which=1)."""
    hk, d = w.num_kv_heads, w.head_dim
    if w.kv_dist == "normal":
        return torch.ones(hk, d)
    g = _gen(w.seed, _T_SCALE, layer, which)
    s = torch.exp(0.5 * torch.randn(hk, d, generator=g))
    for h in range(hk):
        if w.n_outliers > 0:
            ch = torch.randperm(d, generator=g)[: w.n_outliers]
            s[h, ch] *= w.outlier_gain
    return s


def make_layer_inputs(w: Workload, lay: BatchLayout, layer: int) -> LayerInputs:
    hk, hq, d = w.num_kv_heads, w.num_q_heads, w.head_dim
    dt = w.torch_dtype
    sk, sv = _scales(w, layer, 0), _scales(w, layer, 1)
    ck, cv = [], []
    for c, n in enumerate(lay.chunk_len):
        gk = _gen(w.seed, _T_K, layer, c)
        gv = _gen(w.seed, _T_V, layer, c)
        ck.append((torch.randn(n, hk, d, generator=gk) * sk).to(dt))
        cv.append((torch.randn(n, hk, d, generator=gv) * sv).to(dt))
    tq = lay.total_q
    q = torch.randn(tq, hq, d, generator=_gen(w.seed, _T_Q, layer)).to(dt)
    kq = (torch.randn(tq, hk, d, generator=_gen(w.seed, _T_KQ, layer)) * sk).to(dt)
    vq = (torch.randn(tq, hk, d, generator=_gen(w.seed, _T_VQ, layer)) * sv).to(dt)
    return LayerInputs(chunk_k=ck, chunk_v=cv, q=q, kq=kq, vq=vq)


@dataclass
class RecomputeInputs:
    """One layer's inputs of the selective recompute.

    x: hidden states of the batch's doc tokens [total_doc, d_model] (request
    order, then position), N(0, 1); w_k, w_v: projection weights
    [H_kv * head_dim, d_model] (a linear layer's layout), N(0, 1 / d_model), so
    that a projected value is about N(0, 1); all rounded once to bf16.
    """
    x: torch.Tensor
    w_k: torch.Tensor
    w_v: torch.Tensor


def make_recompute_inputs(w: Workload, lay: BatchLayout, layer: int, rows: int = None) -> RecomputeInputs:
    """rows: hidden-state rows to draw (default: one per doc token of the batch;
    fewer when the caller indexes them by selection rank)."""
    n_out = w.num_kv_heads * w.head_dim
    std = 1.0 / float(w.d_model) ** 0.5
    n_rows = lay.total_doc if rows is None else rows
    x = torch.randn(n_rows, w.d_model, generator=_gen(w.seed, _T_X, layer)).to(torch.bfloat16)
    wk = (torch.randn(n_out, w.d_model, generator=_gen(w.seed, _T_WK, layer)) * std).to(torch.bfloat16)
    wv = (torch.randn(n_out, w.d_model, generator=_gen(w.seed, _T_WV, layer)) * std).to(torch.bfloat16)
    return RecomputeInputs(x=x, w_k=wk, w_v=wv)


def random_selection(doc_lens, counts, seed: int) -> list:
    """Seeded stand-in for a top-k result: per request, counts[b] distinct doc
    positions in random order (a selection lists positions by impact rank,
    which is unrelated to position order)."""
    g = _gen(seed, 123)
    out = []
    for n, k in zip(doc_lens, counts):
        k = min(int(k), int(n))
        out.append(torch.randperm(int(n), generator=g)[:k].tolist() if n > 0 else [])
    return out


@dataclass
class EncodedLayer:
    """A synthetic quantized stream of every distinct chunk of one layer: random
    b-bit codes [total_tokens][H_kv][128 * b / 8] (bytes) for K and V, and per
    chunk, KV head and channel an fp32 scale (lognormal) and offset (normal)."""
    bits: int
    codes_k: torch.Tensor
    codes_v: torch.Tensor
    scale_k: torch.Tensor
    offset_k: torch.Tensor
    scale_v: torch.Tensor
    offset_v: torch.Tensor


def make_encoded_layer(w: Workload, lay: BatchLayout, layer: int, bits: int) -> EncodedLayer:
    g = _gen(w.seed, _T_CODES, layer)
    n = sum(lay.chunk_len)
    row = w.head_dim * bits // 8
    nc = len(lay.chunk_len)
    codes = lambda: torch.randint(0, 256, (n, w.num_kv_heads, row), generator=g, dtype=torch.int32).to(torch.uint8)
    scale = lambda: torch.exp(0.5 * torch.randn(nc, w.num_kv_heads, w.head_dim, generator=g)) * 0.02
    offset = lambda: -2.0 + 0.5 * torch.randn(nc, w.num_kv_heads, w.head_dim, generator=g)
    return EncodedLayer(bits, codes(), codes(), scale(), offset(), scale(), offset())
