"""Shared helpers of the GPU tests: put a generated workload on the device,
run the library on it, and compare with the oracle."""

from __future__ import annotations

import numpy as np
import torch

import oracle.prefill as orc
from serving_prefill_b200 import Batch, KVPool
from serving_prefill_b200.engine import PrefillEngine, write_chunks
from workloads import make_layer_inputs, make_layout

BF16_ATOL = 1e-2
BF16_RTOL = 1e-2
F32_ATOL = 1e-5
F32_RTOL = 1e-5
IMPACT_RTOL = 1e-3
TIE_RTOL = 1e-4


class DeviceCase:
    """A workload's pool (the given layers), batch and engine on the GPU."""

    def __init__(self, w, lay=None, layers=None, device="cuda", spare_pages=0, transform=None):
        """transform(inputs): optional in-place change of each layer's seeded
        inputs before they are written; the oracle sees the same inputs."""
        self.w = w
        self.lay = make_layout(w) if lay is None else lay
        self.layers = list(range(w.num_layers)) if layers is None else list(layers)
        self.pool = KVPool(w.num_layers, self.lay.num_pages + spare_pages, w.num_kv_heads, w.head_dim,
                           dtype=w.torch_dtype, device=device)
        self.batch = Batch(self.lay.req_chunk_off, self.lay.chunk_doc_off, self.lay.chunk_page_off,
                           self.lay.page_ids, self.lay.q_off, device=device)
        self.engine = PrefillEngine(self.pool, self.batch, w.num_q_heads, w.r, dtype=w.torch_dtype, device=device)
        self.inputs = {}
        self.dev_inputs = {}
        self.err = torch.zeros(1, dtype=torch.int32, device=device)
        pages = [p.to(torch.int32).to(device) for p in self.lay.chunk_pages]
        for layer in self.layers:
            inp = make_layer_inputs(w, self.lay, layer)
            if transform is not None:
                transform(inp)
            self.inputs[layer] = inp
            write_chunks(self.pool, layer, pages, [k.to(device) for k in inp.chunk_k],
                         [v.to(device) for v in inp.chunk_v], device_err=self.err)
            self.dev_inputs[layer] = (inp.q.to(device), inp.kq.to(device), inp.vq.to(device))
        torch.cuda.synchronize()

    def run_layer(self, layer, with_impact):
        q, kq, vq = self.dev_inputs[layer]
        self.engine.attend(layer, q, kq, vq, with_impact=with_impact)
        if with_impact:
            self.engine.select()
        torch.cuda.synchronize()
        e = self.engine
        out = {
            "o": e.o[: self.batch.total_q].float().cpu().double().numpy(),
            "lse": e.row_lse[: self.batch.total_q].cpu().double().numpy(),
        }
        if with_impact:
            out["impact"] = e.impact[: self.batch.total_doc + self.batch.total_q].cpu().double().numpy()
            out["topk_idx"] = e.topk_idx.cpu().numpy()
            out["topk_val"] = e.topk_val.cpu().numpy()
            out["k"] = e.k.cpu().numpy()
        return out

    def oracle(self, layer, with_impact):
        return orc.run_workload_layer(self.lay, self.inputs[layer], want_impact=with_impact)


def assert_o_close(got, ref, dtype):
    atol, rtol = (BF16_ATOL, BF16_RTOL) if dtype == "bf16" else (F32_ATOL, F32_RTOL)
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    bad = err > bound
    assert not bad.any(), (f"O mismatch at {np.argwhere(bad)[:5].tolist()} "
                           f"max err {err.max():.3g}, worst ratio {(err / bound).max():.3g}")


def assert_lse_close(got, ref_m, ref_l, dtype):
    ref = ref_m + np.log(ref_l)
    tol = 2e-3 if dtype == "bf16" else 1e-5
    err = np.abs(got - ref)
    assert err.max() <= tol * np.maximum(1.0, np.abs(ref)).max(), f"lse max err {err.max():.3g}"


def assert_impact_close(got, ref):
    rel = np.abs(got - ref) / np.maximum(np.abs(ref), 1e-30)
    assert rel.max() <= IMPACT_RTOL, f"impact max rel err {rel.max():.3g} at {int(rel.argmax())}"


def assert_topk_ok(case_lay, out, ref):
    """Top-k sets equal up to near-ties of the k-th value; order and values valid."""
    at = 0
    for b in range(case_lay.num_requests):
        n_doc = case_lay.doc_lens[b]
        q = case_lay.q_lens[b]
        k = int(out["k"][b])
        kref = len(ref.topk[b])
        assert k == kref, f"request {b}: k {k} != {kref}"
        idx = out["topk_idx"][b][:k]
        assert np.all(out["topk_idx"][b][k:] == -1)
        gimp = out["impact"][at:at + n_doc]
        rimp = ref.impact[at:at + n_doc]
        # exact selection on the GPU's own impact values
        want = sorted(range(n_doc), key=lambda i: (-np.float32(gimp[i]), i))[:k]
        assert idx.tolist() == want, f"request {b}: top-k is not the sorted prefix of the impacts"
        np.testing.assert_array_equal(out["topk_val"][b][:k], gimp[idx].astype(np.float32))
        # set parity with the oracle, near-ties of the k-th value excluded
        if k > 0:
            vk = rimp[ref.topk[b][-1]]
            near = set(np.nonzero(np.abs(rimp - vk) <= TIE_RTOL * vk)[0].tolist())
            assert set(idx.tolist()) - near == set(ref.topk[b].tolist()) - near, f"request {b}: top-k sets differ"
        at += n_doc + q


def check_layer(case, layer, with_impact):
    out = case.run_layer(layer, with_impact)
    ref = case.oracle(layer, with_impact)
    assert_o_close(out["o"], ref.o, case.w.dtype)
    assert_lse_close(out["lse"], ref.m, ref.l, case.w.dtype)
    if with_impact:
        assert_impact_close(out["impact"], ref.impact)
        assert_topk_ok(case.lay, out, ref)
    st, bits = case.engine.device_error()
    assert st == 0 and bits == 0, f"device error {st} bits {bits}"
    return out, ref
