"""RoPE position re-basing on the GPU (rag_fused_prefill_attn_rope) against
the oracle's re-based attention, Impact and top-k (oracle/prefill.py,
step 2b), at the tolerances of the plain path. The cases put chunk
boundaries inside key tiles (short chunks), use several requests, GQA groups
of 1 to 8, and the full-size 32-layer Llama-3-8B layer and 70B-shaped layer
with their rotary bases."""

import numpy as np
import pytest
import torch

from serving_prefill_b200.rag import rag_fused_prefill_attn_rope
from workloads import get_workload, scaled

from gpu_support import (DeviceCase, assert_impact_close, assert_lse_close, assert_o_close, assert_topk_ok)

pytestmark = pytest.mark.gpu


def run_rope(case, layer, base):
    e = case.engine
    q, kq, vq = case.dev_inputs[layer]
    rag_fused_prefill_attn_rope(case.pool, layer, case.batch, q, kq, vq, e.o, e.ws, base, impact=e.impact,
                                row_lse=e.row_lse)
    e.select()
    torch.cuda.synchronize()
    b = case.batch
    return {"o": e.o[: b.total_q].float().cpu().double().numpy(),
            "lse": e.row_lse[: b.total_q].cpu().double().numpy(),
            "impact": e.impact[: b.total_doc + b.total_q].cpu().double().numpy(),
            "topk_idx": e.topk_idx.cpu().numpy(), "topk_val": e.topk_val.cpu().numpy(), "k": e.k.cpu().numpy()}


def check_rope(w, base, layer=0):
    case = DeviceCase(w, layers=[layer])
    out = run_rope(case, layer, base)
    import oracle.prefill as orc
    ref = orc.run_workload_layer(case.lay, case.inputs[layer], want_impact=True, rope_base=base)
    assert_o_close(out["o"], ref.o, "bf16")
    assert_lse_close(out["lse"], ref.m, ref.l, "bf16")
    assert_impact_close(out["impact"], ref.impact)
    assert_topk_ok(case.lay, out, ref)
    st, bits = case.engine.device_error()
    assert st == 0 and bits == 0, (st, bits)
    return out, ref


def small_cases():
    l3 = get_workload("llama3_8b_l32")
    b16 = get_workload("batched16")
    l2 = get_workload("llama2_7b_l1")
    return {
        "short_chunks_gqa4": (scaled(l3, num_layers=1, num_q_heads=8, num_kv_heads=2,
                                     chunk_lens=(40, 70, 1, 33, 300, 17), q_len=30), 500000.0),
        "pooled": (scaled(b16, num_q_heads=8, num_kv_heads=2, n_requests=5, n_pool_chunks=12,
                          chunk_len_range=(1, 400), chunks_per_req=(1, 4), q_range=(1, 90)), 500000.0),
        "mha_llama2_base": (scaled(l2, num_q_heads=4, num_kv_heads=4, chunk_lens=(200, 77, 300), q_len=40),
                            10000.0),
        "g8_split": (scaled(get_workload("long70b"), num_q_heads=16, num_kv_heads=2, chunk_lens=(700,) * 6,
                            q_len=150), 500000.0),
    }


CASES = small_cases()


@pytest.mark.parametrize("name", list(CASES))
def test_rope_parity_small(name):
    w, base = CASES[name]
    check_rope(w, base)


def test_rope_changes_the_result():
    """Re-basing is not the identity once a request holds more than one chunk."""
    w, base = CASES["short_chunks_gqa4"]
    case = DeviceCase(w, layers=[0])
    a = run_rope(case, 0, base)
    b = case.run_layer(0, True)
    assert not np.allclose(a["o"], b["o"], atol=1e-2, rtol=1e-2)


@pytest.mark.slow
@pytest.mark.parametrize("name,base", [("llama3_8b_l32", 500000.0), ("long70b", 500000.0)])
def test_rope_parity_full_size(name, base):
    w = get_workload(name)
    check_rope(w, base, layer=w.impact_layer_index)
