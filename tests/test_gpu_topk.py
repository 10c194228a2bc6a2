"""The top-k kernel alone, through the C ABI, on seeded impact vectors.

It is a pure function of the impact vector, so it is checked bit-exactly
against the oracle's stable sort on the same fp32 values: the whole-sort path
(short requests), the bucket-candidate path (long requests) and the exact
fallback when one bucket holds more candidates than fit in shared memory
(mass ties, all-zero impacts).
"""

import numpy as np
import pytest
import torch

import oracle.prefill as orc
from serving_prefill_b200 import Batch, rag_impact_topk, rag_recompute_count

pytestmark = pytest.mark.gpu


def run_topk(segments, r):
    n = [len(s) for s in segments]
    pages = [-(-x // 16) for x in n]
    batch = Batch(req_chunk_off=list(range(len(n) + 1)), chunk_doc_off=np.cumsum([0] + n).tolist(),
                  chunk_page_off=np.cumsum([0] + pages).tolist(), page_ids=list(range(sum(pages))),
                  q_off=[0] * (len(n) + 1))
    impact = torch.from_numpy(np.concatenate(segments).astype(np.float32)).cuda()
    k_cap = max(1, max(rag_recompute_count(x, r) for x in n))
    idx = torch.empty(len(n), k_cap, dtype=torch.int32, device="cuda")
    val = torch.empty(len(n), k_cap, dtype=torch.float32, device="cuda")
    kk = torch.empty(len(n), dtype=torch.int32, device="cuda")
    rag_impact_topk(impact, batch, r, k_cap, idx, val, kk)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), val.cpu().numpy(), kk.cpu().numpy()


def check(segments, r):
    idx, val, kk = run_topk(segments, r)
    for b, seg in enumerate(segments):
        seg32 = seg.astype(np.float32)
        k = orc.recompute_count(len(seg), r) if len(seg) else 0
        assert kk[b] == k
        want = orc.select_topk(seg32.astype(np.float64), k)
        assert idx[b, :k].tolist() == want.tolist(), f"request {b} (n={len(seg)})"
        np.testing.assert_array_equal(val[b, :k], seg32[want])
        assert np.all(idx[b, k:] == -1)


def test_short_requests_whole_sort():
    rng = np.random.default_rng(1)
    check([rng.random(n) for n in (1, 5, 120, 2048, 8192)], 0.1)


def test_long_request_bucket_path():
    rng = np.random.default_rng(2)
    check([rng.lognormal(-6, 1.0, 65536), rng.random(20000), rng.lognormal(0, 0.01, 9000)], 0.05)


def test_mass_ties_fall_back_to_exact_select():
    rng = np.random.default_rng(3)
    few_values = rng.integers(0, 4, 60000).astype(np.float64) / 3.0   # 4 distinct values, ~15k each
    check([few_values, np.zeros(65536), np.full(10000, 0.25)], 0.1)


def test_k_one_and_large_ratio():
    rng = np.random.default_rng(4)
    check([rng.random(15), rng.random(9)], 0.1)          # k = 1
    check([rng.random(12000)], 0.6)                       # k = 7200


def test_cluster_of_four_ctas():
    rng = np.random.default_rng(5)
    check([rng.lognormal(-5, 1.5, 30000), rng.random(100)], 0.1)   # longest 30,000: four CTAs per request


def test_buckets_at_the_rank_limit():
    # one 12-bit bucket of 256 keys (ordered by counting) above one of 257 keys
    # (ordered by a sorting network), both inside the top k
    rng = np.random.default_rng(6)
    y = 1.25 + 0.125 * rng.random(256)        # [1.25, 1.375): one bucket
    x = 1.0 + 0.125 * rng.random(257)         # [1.0, 1.125): the bucket below it
    low = 0.5 * rng.random(5000)
    seg = np.concatenate([low[:2000], y, low[2000:], x])
    n = len(seg)
    check([seg], 600.5 / n)                    # k = 600: both buckets and 87 lower keys


def test_large_buckets_use_wide_sorts():
    rng = np.random.default_rng(7)
    check([rng.random(65536)], 0.1)            # buckets of ~4,096 keys
    check([rng.random(131072)], 0.05)          # the top bucket holds ~8,192 keys


def test_many_buckets_across_the_cluster():
    rng = np.random.default_rng(8)
    check([rng.lognormal(-6, 2.5, 65536)], 0.1)   # hundreds of buckets dealt over eight CTAs


def test_k_above_eight_thousand():
    # 65,536 doc tokens at r = 0.15, inside the pages' 0.05-0.15 range: k = 9,830
    rng = np.random.default_rng(9)
    check([rng.lognormal(-6, 1.0, 65536)], 0.15)
    check([rng.random(65536), rng.random(300)], 0.15)


def test_k_at_the_limit():
    # k = int(109,227 * 0.15) = 16,384, the largest selection a request may make
    rng = np.random.default_rng(10)
    n = 109227
    assert rag_recompute_count(n, 0.15) == 16384
    check([rng.lognormal(-5, 1.2, n)], 0.15)


def test_bucket_above_the_kth_longer_than_a_register_sort():
    # 10,000 keys in one 12-bit bucket above the k-th key's bucket: that segment
    # is longer than the 8,192 keys the register sorting networks hold
    rng = np.random.default_rng(11)
    a = 2.0 + 0.25 * rng.random(10000)        # [2, 2.25): one bucket
    b = 1.0 + 0.125 * rng.random(10000)       # [1, 1.125): the bucket below it
    low = 0.5 * rng.random(80000)
    seg = np.concatenate([low[:40000], a, low[40000:], b])
    n = len(seg)
    check([seg], 12000.5 / n)                  # k = 12,000: all of a, 2,000 of b


def test_whole_sort_boundary():
    # 4,096 doc tokens are sorted whole by one CTA; 4,097 take the bucket path
    rng = np.random.default_rng(12)
    check([rng.random(4096), rng.lognormal(-4, 1.0, 4097), rng.integers(0, 3, 4096).astype(np.float64)], 0.15)


def test_one_cta_counting_limits():
    # A request of at most 8,192 doc tokens is ordered by counting inside its
    # 12-bit buckets when at most 1,024 keys lie in the k-th key's bucket or
    # above and their squared bucket lengths add up to at most 131,072;
    # otherwise it takes the general path. The top keys are drawn inside
    # chosen buckets (fp32 bit patterns with fixed top 12 bits, from 2.0 up),
    # the rest below 0.5; k takes all top keys but one.
    rng = np.random.default_rng(13)
    low = 0.5 * rng.random(3000)

    def buckets(sizes):
        parts = [((np.uint32(1024 + j) << np.uint32(20)) | rng.integers(0, 1 << 20, c).astype(np.uint32))
                 for j, c in enumerate(sizes)]
        return np.concatenate(parts).view(np.float32).astype(np.float64)

    for sizes in ([256, 147, 147, 149],        # 131,019 comparisons: counting
                  [256, 147, 147, 150],        # 131,254: general path
                  [64] * 16,                   # 1,024 keys: counting
                  [64] * 15 + [65],            # 1,025 keys (65,665 comparisons): general path
                  [362], [363],                # one bucket: 131,044 counting, 131,769 general
                  [40, 3, 100, 0, 77]):        # short buckets
        top = buckets(sizes)
        seg = np.concatenate([low[:1500], top, low[1500:]])
        check([seg], (len(top) - 0.5) / len(seg))
    tied = np.concatenate([low, np.full(200, 1.0), low[:100]])
    check([tied, rng.random(7000)], 0.05)           # 200 equal keys above the rest; uniform keys
