"""rag_fused_prefill_attn_static: the entry point for callers that cannot
allocate device memory.

Such callers (a runtime that hands a plugin only its input and output buffers,
a deployment whose device memory is planned once at start-up) cannot provide
the workspace rag_fused_prefill_attn needs; this entry point runs the same
computation in the library's fixed 64 MiB device array. The test calls it
through the C ABI twice in a row and compares each result with the workspace
entry point's, within the tolerances the parity tests use. It lives in its own
file so that pytest collects it last, and it passes alone in a fresh process
as well as after the other tests.
"""

import numpy as np
import pytest
import torch

from serving_prefill_b200.rag import rag_fused_prefill_attn_static
from workloads import get_workload, scaled

from gpu_support import DeviceCase, assert_impact_close, assert_o_close

pytestmark = pytest.mark.gpu


def _cases():
    b16 = get_workload("batched16")
    l70 = get_workload("long70b")
    return {
        # several requests, short key ranges: one split per unit (direct epilogue)
        "pooled": scaled(b16, num_q_heads=8, num_kv_heads=2, n_requests=5, n_pool_chunks=12,
                         chunk_len_range=(1, 400), chunks_per_req=(1, 4), q_range=(1, 90)),
        # long key range: split-KV partials in the scratch array, then the combine
        "split": scaled(l70, num_q_heads=16, num_kv_heads=2, chunk_lens=(2048,) * 6, q_len=150),
        # decode step (one token, 4 rows per unit): the decode kernel
        "decode": scaled(get_workload("decode16"), num_q_heads=8, num_kv_heads=2, n_requests=6, n_pool_chunks=10,
                         chunk_len_range=(100, 900), chunks_per_req=(2, 4), context_range=(1, 200)),
    }


@pytest.mark.parametrize("name", ["pooled", "split", "decode"])
def test_static_scratch_matches_workspace_entry(name):
    w = _cases()[name]
    case = DeviceCase(w, layers=[0])
    ref = case.run_layer(0, True)                       # workspace entry point
    q, kq, vq = case.dev_inputs[0]
    tq = case.batch.total_q
    n_imp = case.batch.total_doc + tq
    for call in range(2):
        o = torch.full_like(case.engine.o, float("nan"))
        lse = torch.full_like(case.engine.row_lse, float("nan"))
        impact = torch.full((max(n_imp, 1),), float("nan"), dtype=torch.float32, device=o.device)
        err = torch.full((1,), -1, dtype=torch.int32, device=o.device)
        rag_fused_prefill_attn_static(case.pool, 0, case.batch, q, kq, vq, o, impact=impact, row_lse=lse,
                                      device_err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0, f"call {call}: device error bits {int(err.item())}"
        assert_o_close(o[:tq].float().cpu().double().numpy(), ref["o"], "bf16")
        np.testing.assert_allclose(lse[:tq].cpu().double().numpy(), ref["lse"], rtol=0, atol=2e-3)
        assert_impact_close(impact[:n_imp].cpu().double().numpy(), ref["impact"])
