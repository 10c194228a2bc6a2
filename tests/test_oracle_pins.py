"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each check names what fixes the expected value: a library routine on a special
case (numpy concatenate, torch scaled_dot_product_attention, sorting), a closed
form (uniform softmax, harmonic sums), an invariant (rows of the weights sum to
one, impacts add up to the query length, chunk-order equivariance, GQA equals
MHA with repeated heads), a hand-worked example (tests/golden) or exact rational
arithmetic. The mutation tests at the end plant plausible mistakes in the
oracle and check that some pin fails.
"""

import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle.prefill as orc
from workloads import get_workload, make_layer_inputs, make_layout, scaled

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def small_pooled():
    w = scaled(get_workload("batched16"), name="pooled_small", n_requests=3, n_pool_chunks=6,
               chunk_len_range=(5, 40), chunks_per_req=(2, 4), q_range=(3, 9),
               num_q_heads=4, num_kv_heads=2, head_dim=16)
    return w


def small_fixed_gqa():
    return scaled(get_workload("long70b"), name="fixed_small", chunk_lens=(17, 5, 30),
                  q_len=6, num_q_heads=8, num_kv_heads=2, head_dim=16)


# ---------------------------------------------------------------- gather

def check_gather_is_concatenation(w):
    lay = make_layout(w)
    inp = make_layer_inputs(w, lay, 0)
    bits = np.uint16 if w.dtype == "bf16" else np.uint32
    pk, _ = orc.build_layer_pool(lay, inp, bits)
    for cs in lay.req_chunks:
        got = orc.gather(pk, 0, [(lay.chunk_pages[c].numpy(), lay.chunk_len[c]) for c in cs])
        want = np.concatenate([orc.to_bits(inp.chunk_k[c]) for c in cs], axis=0)
        assert got.dtype == want.dtype and np.array_equal(got, want)


@pytest.mark.parametrize("wname", ["tiny", "pooled", "gqa"])
def test_gather_is_concatenation(wname):
    w = {"tiny": get_workload("tiny"), "pooled": small_pooled(), "gqa": small_fixed_gqa()}[wname]
    check_gather_is_concatenation(w)


def test_gather_ignores_physical_placement():
    w = small_pooled()
    lay = make_layout(w)
    lay2 = lay.with_page_permutation(seed=5)
    assert not all(torch.equal(a, b) for a, b in zip(lay.chunk_pages, lay2.chunk_pages))
    inp = make_layer_inputs(w, lay, 0)
    p1, _ = orc.build_layer_pool(lay, inp, np.uint16)
    p2, _ = orc.build_layer_pool(lay2, inp, np.uint16)
    for cs in lay.req_chunks:
        g1 = orc.gather(p1, 0, [(lay.chunk_pages[c].numpy(), lay.chunk_len[c]) for c in cs])
        g2 = orc.gather(p2, 0, [(lay2.chunk_pages[c].numpy(), lay2.chunk_len[c]) for c in cs])
        assert np.array_equal(g1, g2)


def test_pool_tail_slots_are_zero():
    w = small_pooled()
    lay = make_layout(w)
    inp = make_layer_inputs(w, lay, 0)
    pk, pv = orc.build_layer_pool(lay, inp, np.uint16)
    for c, n in enumerate(lay.chunk_len):
        last = int(lay.chunk_pages[c][-1])
        used = n - 16 * (len(lay.chunk_pages[c]) - 1)
        assert np.all(pk[0, last, :, used:, :] == 0) and np.all(pv[0, last, :, used:, :] == 0)


# ---------------------------------------------------------------- attention

def _request_inputs(w, lay, inp, b):
    q0 = sum(lay.q_lens[:b])
    ql = lay.q_lens[b]
    cs = lay.req_chunks[b]
    kd = np.concatenate([orc.to_f64(inp.chunk_k[c]) for c in cs], axis=0)
    vd = np.concatenate([orc.to_f64(inp.chunk_v[c]) for c in cs], axis=0)
    kcat = np.concatenate([kd, orc.to_f64(inp.kq[q0:q0 + ql])], axis=0)
    vcat = np.concatenate([vd, orc.to_f64(inp.vq[q0:q0 + ql])], axis=0)
    return orc.to_f64(inp.q[q0:q0 + ql]), kcat, vcat, kd.shape[0]


def check_attention_vs_sdpa(w):
    """torch fp64 scaled_dot_product_attention with an explicit boolean mask."""
    lay = make_layout(w)
    inp = make_layer_inputs(w, lay, 0)
    for b in range(lay.num_requests):
        q, kcat, vcat, n_doc = _request_inputs(w, lay, inp, b)
        o, m, l, imp, _ = orc.attend_request(q, kcat, vcat, n_doc, 1.0 / math.sqrt(w.head_dim))
        ql, n_tot = q.shape[0], kcat.shape[0]
        G = w.num_q_heads // w.num_kv_heads
        qt = torch.from_numpy(q).permute(1, 0, 2)                     # [H, q, d]
        kt = torch.from_numpy(kcat).permute(1, 0, 2).repeat_interleave(G, dim=0)
        vt = torch.from_numpy(vcat).permute(1, 0, 2).repeat_interleave(G, dim=0)
        keep = torch.ones(ql, n_tot, dtype=torch.bool).tril(diagonal=n_doc)
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=keep)
        np.testing.assert_allclose(o, ref.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("wname", ["tiny", "pooled", "gqa"])
def test_attention_vs_sdpa(wname):
    w = {"tiny": get_workload("tiny"), "pooled": small_pooled(), "gqa": small_fixed_gqa()}[wname]
    check_attention_vs_sdpa(w)


def check_rows_sum_to_one_and_mask():
    w = small_fixed_gqa()
    lay = make_layout(w)
    inp = make_layer_inputs(w, lay, 0)
    q, kcat, vcat, n_doc = _request_inputs(w, lay, inp, 0)
    o, m, l, imp, alpha = orc.attend_request(q, kcat, vcat, n_doc, 1 / 4.0, want_alpha=True)
    np.testing.assert_allclose(alpha.sum(axis=2), 1.0, rtol=0, atol=1e-12)
    for j in range(q.shape[0]):
        assert np.all(alpha[:, j, n_doc + j + 1:] == 0)
        assert np.all(alpha[:, j, : n_doc + j + 1] > 0)


def test_rows_sum_to_one_and_mask():
    check_rows_sum_to_one_and_mask()


def check_uniform_closed_form(n_doc=37, ql=5, hq=4, hk=2, d=8):
    """Q = 0: every visible key has weight 1 / (n_doc + j + 1)."""
    rng = np.random.default_rng(3)
    q = np.zeros((ql, hq, d))
    kcat = rng.standard_normal((n_doc + ql, hk, d))
    vcat = rng.standard_normal((n_doc + ql, hk, d))
    o, m, l, imp, _ = orc.attend_request(q, kcat, vcat, n_doc, 0.3)
    G = hq // hk
    for j in range(ql):
        for h in range(hq):
            want = vcat[: n_doc + j + 1, h // G, :].mean(axis=0)
            np.testing.assert_allclose(o[j, h], want, rtol=1e-12, atol=1e-13)
    harm = lambda n: sum(Fraction(1, t) for t in range(1, n + 1))  # noqa: E731
    doc_val = float(harm(n_doc + ql) - harm(n_doc))
    np.testing.assert_allclose(imp[:n_doc], doc_val, rtol=1e-12)
    for t in range(ql):
        want = float(sum(Fraction(1, n_doc + j + 1) for j in range(t, ql)))
        np.testing.assert_allclose(imp[n_doc + t], want, rtol=1e-12)
    np.testing.assert_allclose(l, (n_doc + np.arange(ql) + 1)[:, None] * np.ones((1, hq)), rtol=1e-12)


def test_uniform_closed_form():
    check_uniform_closed_form()


def check_one_hot():
    """A key aligned with the query at large norm takes all of the weight."""
    rng = np.random.default_rng(4)
    n_doc, ql, d = 20, 3, 8
    q = rng.standard_normal((ql, 1, d))
    kcat = rng.standard_normal((n_doc + ql, 1, d)) * 0.01
    vcat = rng.standard_normal((n_doc + ql, 1, d))
    for j in range(ql):
        kcat[7 + j, 0] = 500.0 * q[j, 0] / np.linalg.norm(q[j, 0])
    o, *_ = orc.attend_request(q, kcat, vcat, n_doc, 1.0)
    for j in range(ql):
        np.testing.assert_allclose(o[j, 0], vcat[7 + j, 0], rtol=1e-9, atol=1e-9)


def test_one_hot():
    check_one_hot()


def check_impact_total_is_q(w):
    lay = make_layout(w)
    inp = make_layer_inputs(w, lay, 0)
    res = orc.run_workload_layer(lay, inp, want_impact=True)
    at = 0
    for b in range(lay.num_requests):
        n = lay.doc_lens[b] + lay.q_lens[b]
        np.testing.assert_allclose(res.impact[at:at + n].sum(), lay.q_lens[b], rtol=1e-9)
        at += n
    assert at == len(res.impact)


@pytest.mark.parametrize("wname", ["tiny", "pooled", "gqa"])
def test_impact_total_is_q(wname):
    w = {"tiny": get_workload("tiny"), "pooled": small_pooled(), "gqa": small_fixed_gqa()}[wname]
    check_impact_total_is_q(w)


def check_chunk_order_equivariance():
    w = small_fixed_gqa()
    lay = make_layout(w)
    inp = make_layer_inputs(w, lay, 0)
    order = [2, 0, 1]
    lay2 = lay.with_chunk_order([order])
    r1 = orc.run_workload_layer(lay, inp, want_impact=True)
    r2 = orc.run_workload_layer(lay2, inp, want_impact=True)
    np.testing.assert_allclose(r1.o, r2.o, rtol=1e-11, atol=1e-12)
    # logical position of each (chunk, token) in either order
    starts1 = np.cumsum([0] + [lay.chunk_len[c] for c in lay.req_chunks[0]])
    starts2 = np.cumsum([0] + [lay2.chunk_len[c] for c in lay2.req_chunks[0]])
    n_doc = lay.doc_lens[0]
    for pos2, c in enumerate(lay2.req_chunks[0]):
        pos1 = lay.req_chunks[0].index(c)
        n = lay.chunk_len[c]
        np.testing.assert_allclose(r2.impact[starts2[pos2]:starts2[pos2] + n],
                                   r1.impact[starts1[pos1]:starts1[pos1] + n], rtol=1e-11)
    np.testing.assert_allclose(r2.impact[n_doc:], r1.impact[n_doc:], rtol=1e-11)


def test_chunk_order_equivariance():
    check_chunk_order_equivariance()


def check_gqa_equals_repeated_mha():
    rng = np.random.default_rng(6)
    n_doc, ql, hq, hk, d = 30, 4, 8, 2, 16
    q = rng.standard_normal((ql, hq, d))
    kcat = rng.standard_normal((n_doc + ql, hk, d))
    vcat = rng.standard_normal((n_doc + ql, hk, d))
    o1, m1, l1, i1, _ = orc.attend_request(q, kcat, vcat, n_doc, 0.25)
    G = hq // hk
    o2, m2, l2, i2, _ = orc.attend_request(q, np.repeat(kcat, G, axis=1), np.repeat(vcat, G, axis=1),
                                           n_doc, 0.25)
    np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(i1, i2, rtol=1e-13)


def test_gqa_equals_repeated_mha():
    check_gqa_equals_repeated_mha()


# ---------------------------------------------------------------- hand example

def _val(s):
    s = str(s)
    if s == "masked":
        return None
    env = {"sqrt": math.sqrt, "ln": math.log, "ln2": math.log(2), "ln3": math.log(3)}
    if "/" in s and "(" not in s:
        return float(Fraction(s))
    return float(eval(s, {"__builtins__": {}}, env))


def check_hand_example():
    g = json.load(open(os.path.join(GOLDEN, "hand_example.json")))
    n_doc = g["n_doc"]
    kcat = np.array(g["k_doc"] + g["k_query"], dtype=np.float64)[:, None, :]
    vcat = np.array(g["v_doc"] + g["v_query"], dtype=np.float64)[:, None, :]
    q = np.array([[_val(x) for x in row] for row in g["q"]])[:, None, :]
    o, m, l, imp, alpha = orc.attend_request(q, kcat, vcat, n_doc, 1 / math.sqrt(2), want_alpha=True)
    np.testing.assert_allclose(alpha[0], [[_val(x) for x in row] for row in g["alpha"]], atol=1e-14)
    np.testing.assert_allclose(o[:, 0], [[_val(x) for x in row] for row in g["o"]], atol=1e-14)
    np.testing.assert_allclose(m[:, 0], [_val(x) for x in g["m"]], atol=1e-14)
    np.testing.assert_allclose(l[:, 0], [_val(x) for x in g["l"]], atol=1e-13)
    np.testing.assert_allclose(imp, [_val(x) for x in g["impact"]], atol=1e-14)
    np.testing.assert_allclose(imp.sum(), _val(g["impact_total"]), atol=1e-14)
    k = orc.recompute_count(n_doc, g["r"])
    assert k == g["k"]
    assert orc.select_topk(imp[:n_doc], k).tolist() == g["topk"]


def test_hand_example():
    check_hand_example()


# ---------------------------------------------------------------- k and top-k

def test_recompute_count_golden():
    g = json.load(open(os.path.join(GOLDEN, "recompute_counts.json")))
    for c in g["cases"]:
        assert orc.recompute_count(c["n_doc"], float(c["r"])) == c["k"], c


def test_recompute_count_of_an_empty_doc_slice_is_zero():
    """A request with no doc tokens has nothing to select (the max(1, .) floor
    applies to a non-empty slice); the selection of such a request is empty."""
    for r in (0.05, 0.1, 0.15, 0.99):
        assert orc.recompute_count(0, r) == 0
        assert orc.select_topk(np.zeros(0), orc.recompute_count(0, r)).tolist() == []


@pytest.mark.parametrize("r", ["0.05", "0.1", "0.15"])
def test_recompute_count_is_exact_floor(r):
    """int(N * r) in double equals floor(N * r) over the exact decimal r."""
    fr = Fraction(r)
    for n in range(1, 20001):
        assert orc.recompute_count(n, float(r)) == max(1, (n * fr.numerator) // fr.denominator)


def check_topk_is_sorted_prefix():
    rng = np.random.default_rng(7)
    for n, k in [(1, 1), (10, 3), (100, 12), (1000, 150), (4096, 4096)]:
        vals = rng.integers(0, 20, n).astype(np.float64) / 7.0   # many exact ties
        got = orc.select_topk(vals, k).tolist()
        want = sorted(range(n), key=lambda i: (-vals[i], i))[:k]
        assert got == want
        tv, _ = torch.topk(torch.from_numpy(vals), k)
        np.testing.assert_array_equal(vals[got], tv.numpy())


def test_topk_is_sorted_prefix():
    check_topk_is_sorted_prefix()


# ---------------------------------------------------------------- mutations

def test_mutation_off_by_one_mask_is_caught(monkeypatch):
    monkeypatch.setattr(orc, "visible", lambda i, j, n_doc: i < n_doc + j)
    with pytest.raises(AssertionError):
        check_uniform_closed_form()
    with pytest.raises(AssertionError):
        check_attention_vs_sdpa(small_fixed_gqa())


def test_mutation_unmasked_softmax_is_caught(monkeypatch):
    monkeypatch.setattr(orc, "visible", lambda i, j, n_doc: np.ones(np.broadcast(i, j).shape, bool))
    with pytest.raises(AssertionError):
        check_uniform_closed_form()


def test_mutation_wrong_kv_head_is_caught(monkeypatch):
    monkeypatch.setattr(orc, "kv_head_of", lambda h, G: h % 2)
    with pytest.raises(AssertionError):
        check_attention_vs_sdpa(small_fixed_gqa())


def test_mutation_topk_order_is_caught(monkeypatch):
    monkeypatch.setattr(orc, "select_topk",
                        lambda imp, k: np.argsort(-np.asarray(imp), kind="quicksort")[::-1][:k])
    with pytest.raises(AssertionError):
        check_topk_is_sorted_prefix()


def test_mutation_gather_slot_is_caught(monkeypatch):
    real = orc.gather

    def bad(pool, layer, chunks):
        return real(pool, layer, [(p[::-1].copy(), n) for p, n in chunks])
    monkeypatch.setattr(orc, "gather", bad)
    with pytest.raises(AssertionError):
        check_gather_is_concatenation(small_pooled())


def test_mutation_impact_over_rows_is_caught(monkeypatch):
    """Summing over keys instead of query rows breaks the closed form and the total."""
    real = orc.attend_request

    def bad(q, kcat, vcat, n_doc, scale, want_impact=True, want_alpha=False):
        o, m, l, imp, a = real(q, kcat, vcat, n_doc, scale, want_impact, True)
        imp = np.zeros(kcat.shape[0])
        imp[: q.shape[0]] = a.sum(axis=(0, 2)) / a.shape[0]
        return o, m, l, imp, (a if want_alpha else None)
    monkeypatch.setattr(orc, "attend_request", bad)
    with pytest.raises(AssertionError):
        check_uniform_closed_form()
