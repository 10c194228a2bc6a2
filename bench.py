"""Benchmark of the fused precomputed-KV RAG prefill step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl mine|reference]

A step is one pass of the whole hot path over one batch: the fused attention
of every layer of the workload (paged gather + causal attention), Impact on
the selecting layer, and the top-k recompute selection. The metric is doc-KV
tokens per second (the doc tokens whose cached K/V the step consumes), over
all GPUs. Inputs are seeded synthetic tensors shaped like the pages'
workloads (see workloads/rag.py); the precomputed pool is resident in HBM.

L2 policy: the timed steps rotate over enough independent copies of the
inputs (pool, Q, K_q, V_q, workspace) that each step's working set has left
the 126 MB L2 before it is touched again. Each copy's step is captured once
in a CUDA graph and replayed.

One JSON line is printed by rank 0. The headline is the 32-layer
Llama-3-8B-shaped workload; at one GPU the other workloads (one Llama-2-7B
layer, 16 batched requests, the 70B-shaped long context, a decode step) are
measured in the same run, each with its own roofline, end-to-end number and
oracle baseline, under "per_config". With --impl reference the same metric is
measured for the fp64 CPU oracle on the host cores (a bounded sample per step).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from workloads import get_workload, make_layer_inputs, make_layout  # noqa: E402

DEFAULT_CONFIG = "llama3_8b_l32"
# the other workloads, each measured in the same run and reported under
# "per_config" of the one JSON line (single-GPU runs only)
PER_CONFIG = ["llama2_7b_l1", "batched16", "long70b", "decode16"]
L2_BYTES = 126 * 1024 * 1024
METRIC = "doc-KV tokens/s through fused attn+impact+top-k; % of roofline at 1 B200"


# ----------------------------------------------------------------------------- arithmetic of the roofline

def step_work(w, lay):
    """Algorithmic FLOPs and bytes of one step (method's own work, once)."""
    d, hq, hk, eb = w.head_dim, w.num_q_heads, w.num_kv_heads, w.elem_bytes
    pairs = sum(q * n + q * (q + 1) // 2 for q, n in zip(lay.q_lens, lay.doc_lens))
    attn_flops = 4 * d * hq * pairs                           # QK^T and PV per visible pair
    impact_flops = 2 * d * hq * pairs                         # the impact pass's own QK^T
    kv_doc = 2 * sum(lay.doc_lens) * hk * d * eb              # K and V gathered, per request
    k_doc = kv_doc // 2
    tq = lay.total_q
    qkv = tq * (hq + 2 * hk) * d * eb
    o_bytes = tq * hq * d * eb
    imp_bytes = (lay.total_doc + tq) * 4
    per_layer_attn_bytes = kv_doc + qkv + o_bytes
    impact_bytes = k_doc + tq * (hq + hk) * d * eb + imp_bytes
    L = w.num_layers
    return {
        "attn_flops_per_launch": attn_flops,
        "attn_bytes_per_launch": per_layer_attn_bytes,
        "impact_flops_per_launch": impact_flops,
        "impact_bytes_per_launch": impact_bytes,
        "step_flops": attn_flops * L,
        "step_bytes": per_layer_attn_bytes * L + (imp_bytes * 2 if w.select else 0),
        "doc_tokens": sum(lay.doc_lens),
    }


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained", j["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def _code_only(text: str) -> str:
    """Kernel source without comments or blank lines (a comment edit leaves the code the same)."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = []
    for line in text.splitlines():
        line = re.sub(r"//.*$", "", line).rstrip()
        if line.strip():
            lines.append(line)
    return "\n".join(lines)


# the source file of each timed kernel kind; its digest also covers the
# device-side headers every kernel includes
KERNEL_SOURCE = {"attn": "attn_fwd.cu", "attn_dec": "decode_fwd.cu", "combine": "attn_combine.cu", "impact": "impact.cu", "topk": "topk.cu",
                 "rc_gemm": "recompute.cu", "rc_copy": "recompute.cu", "rc_plan": "recompute.cu",
                 "kv_decode": "kv_decode.cu", "simt_attn": "simt_f32.cu", "simt_impact": "simt_f32.cu"}


def kernel_sources_digest(kernel, read=None):
    """Digest of a kernel's source and the device headers, comments and blank lines removed."""
    read = read or (lambda f: open(os.path.join(ROOT, "serving_prefill_b200", "csrc", f)).read())
    h = hashlib.sha256()
    for f in ("ptx.cuh", "common.cuh", KERNEL_SOURCE.get(kernel, "attn_fwd.cu")):
        h.update(_code_only(read(f)).encode())
    return h.hexdigest()[:16]


def recorded_traffic(config, kernel):
    """DRAM bytes per launch from the committed ncu summary, if it matches these sources."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    j = json.load(open(p))
    e = j.get(f"{config}/{kernel}")
    if not e or e.get("src_digest") != kernel_sources_digest(kernel):
        return None
    return e.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- GPU arm

class Replica:
    """One independent copy of the step's device inputs and buffers."""

    def __init__(self, w, lay, layer_inputs, device):
        from serving_prefill_b200 import Batch, KVPool
        from serving_prefill_b200.engine import PrefillEngine, write_chunks
        self.pool = KVPool(w.num_layers, lay.num_pages, w.num_kv_heads, w.head_dim, dtype=w.torch_dtype,
                           device=device)
        self.batch = Batch(lay.req_chunk_off, lay.chunk_doc_off, lay.chunk_page_off, lay.page_ids, lay.q_off,
                           device=device)
        self.engine = PrefillEngine(self.pool, self.batch, w.num_q_heads, w.r, dtype=w.torch_dtype, device=device)
        pages = [p.to(torch.int32).to(device) for p in lay.chunk_pages]
        self.layers = []
        for layer in range(w.num_layers):
            inp = layer_inputs[layer]
            write_chunks(self.pool, layer, pages, [k.to(device) for k in inp.chunk_k],
                         [v.to(device) for v in inp.chunk_v])
            self.layers.append((layer, inp.q.to(device), inp.kq.to(device), inp.vq.to(device)))
        tq = lay.total_q
        self.outs = [torch.empty(max(tq, 1), w.num_q_heads, w.head_dim, dtype=w.torch_dtype, device=device)
                     for _ in range(w.num_layers)]
        self.impact_layer = w.impact_layer_index
        self.graph = None

    def step(self):
        self.engine.step(self.layers, self.impact_layer, outs=self.outs)

    def capture(self):
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.step()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self.step()
        torch.cuda.synchronize()

    def nbytes(self):
        return self.pool.k.numel() * self.pool.k.element_size() * 2 + sum(
            t.numel() * t.element_size() for _, q, kq, vq in self.layers for t in (q, kq, vq))


def run_gpu(args, w, rank, world, device):
    import serving_prefill_b200 as sp
    torch.cuda.set_device(device)
    lay = make_layout(w)
    layer_inputs = [make_layer_inputs(w, lay, layer) for layer in range(w.num_layers)]
    work = step_work(w, lay)
    first = Replica(w, lay, layer_inputs, device)
    per_copy = first.nbytes()
    n_copies = max(1, min(16, -(-2 * L2_BYTES // per_copy)))
    free = torch.cuda.mem_get_info(device)[0]
    n_copies = max(1, min(n_copies, int(0.5 * free // max(per_copy, 1)) + 1))
    reps = [first] + [Replica(w, lay, layer_inputs, device) for _ in range(n_copies - 1)]
    for r in reps:
        r.step()
    torch.cuda.synchronize()
    st, bits = first.engine.device_error()
    if st != 0:
        raise RuntimeError(f"device error {st} bits {bits}")
    for r in reps:
        r.capture()

    # warm-up
    for i in range(args.warmup):
        reps[i % n_copies].graph.replay()
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    clocks = ClockSampler(device if isinstance(device, int) else torch.cuda.current_device())
    clocks.start()
    time.sleep(0.2)
    barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    for i in range(args.steps):
        reps[i % n_copies].graph.replay()
    ev1.record()
    torch.cuda.synchronize()
    barrier()
    ms = ev0.elapsed_time(ev1)
    # launches inside the timed region: graph replays carry the captured kernels
    per_step_launches = None

    # per-kernel timing pass: the step is captured once more with an event
    # pair around every kernel (event nodes of the graph) and replayed; each
    # replay's device times are read back, so host enqueue latency never
    # enters the per-kernel numbers
    sp.rag_profile_collect()
    sp.rag_profile_enable(True)
    base = sp.rag_launch_count()
    prof_graph = torch.cuda.CUDAGraph()
    s_cap = torch.cuda.Stream()
    s_cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(prof_graph, stream=s_cap):
        first.step()
    per_step_launches = sp.rag_launch_count() - base
    sp.rag_profile_enable(False)
    torch.cuda.synchronize()
    prof_steps = max(3, min(args.steps, 200))
    acc = {}
    timing = "event pairs captured in a CUDA graph with the step"
    try:
        for i in range(prof_steps):
            prof_graph.replay()
            torch.cuda.synchronize()
            for k, (ms_k, n_k) in sp.rag_profile_peek().items():
                a = acc.setdefault(k, [0.0, 0])
                a[0] += ms_k
                a[1] += n_k
        sp.rag_profile_collect()
    except sp.RagError:
        # event nodes not readable: time eager launches instead
        timing = "event pairs around eager launches"
        try:
            sp.rag_profile_collect()
        except sp.RagError:
            pass
        sp.rag_profile_enable(True)
        for i in range(prof_steps):
            reps[i % n_copies].step()
        torch.cuda.synchronize()
        acc = {k: list(v) for k, v in sp.rag_profile_collect().items()}
        sp.rag_profile_enable(False)
    prof = {k: (v[0], v[1]) for k, v in acc.items()}
    del prof_graph
    clk = clocks.stop()

    ms_max = max_over_ranks(ms, world, device)
    ms_per_step = ms_max / args.steps
    value = whole_job_rate(world, work["doc_tokens"], args.steps, ms_max)

    # dominant kernel and its roofline
    peaks = load_peaks()
    kinds = {k: v for k, v in prof.items() if v[1] > 0}
    dom = max(kinds, key=lambda k: kinds[k][0])
    dom_ms, dom_n = kinds[dom]
    avg_s = dom_ms / dom_n / 1e3
    per_launch = {
        "attn": (work["attn_flops_per_launch"], work["attn_bytes_per_launch"]),
        "attn_dec": (work["attn_flops_per_launch"], work["attn_bytes_per_launch"]),
        "combine": (0, 0),
        "impact": (work["impact_flops_per_launch"], work["impact_bytes_per_launch"]),
        "topk": (0, (lay.total_doc + lay.total_q) * 4),
        "simt_attn": (work["attn_flops_per_launch"], work["attn_bytes_per_launch"]),
        "simt_impact": (work["impact_flops_per_launch"], work["impact_bytes_per_launch"]),
    }.get(dom, (0, 0))
    flops, nbytes = per_launch
    long_region = ms > 1000.0
    tflops_peak = peaks["bf16_tflops_sustained"] if long_region else peaks["bf16_tflops"]
    ridge = tflops_peak * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if flops and flops / max(nbytes, 1) > ridge:
        achieved = flops / avg_s / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tflops_peak, "unit": "TFLOP/s",
                "frac": achieved / tflops_peak}
    else:
        achieved = nbytes / avg_s / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"]}
    roof["kernel"] = dom
    roof["peak_source"] = peaks["source"]
    roof["avg_launch_us"] = avg_s * 1e6
    roof["traffic"] = recorded_traffic(w.name, dom)
    t_roof = max(work["step_flops"] / (tflops_peak * 1e12), work["step_bytes"] / (peaks["hbm_gbs"] * 1e9))
    step_roof = {"t_roof_us": t_roof * 1e6, "t_step_us": ms_per_step * 1e3, "frac": t_roof / (ms_per_step / 1e3)}

    # end to end through the public API with host buffers
    e2e = run_e2e(args, w, lay, layer_inputs, first, device, world)

    kernels = {k: {"ms_per_step": v[0] / prof_steps, "launches_per_step": v[1] / prof_steps} for k, v in kinds.items()}
    return {
        "value": value, "ms_per_step": ms_per_step, "roofline": roof, "step_roofline": step_roof,
        "e2e": e2e, "gpu_launches": int(round(per_step_launches * args.steps)), "clocks": clk,
        "kernels": kernels, "copies": n_copies, "work": work, "kernel_timing": timing,
    }


E2E_GROUP = 8   # layers whose inputs (and outputs) move host <-> device in one copy


def run_e2e(args, w, lay, layer_inputs, rep, device, world):
    """Same step through the public API with pinned host inputs and outputs.

    Every step copies the batch descriptors and every layer's q, kq, vq from
    pinned host memory and returns every layer's O (and the top-k) to pinned
    host memory; the engine's HostStep overlaps those copies with the kernels.
    """
    from serving_prefill_b200.engine import HostStep, layer_groups
    eng = rep.engine
    per_layer = [tuple(t.contiguous() for t in (layer_inputs[l].q, layer_inputs[l].kq, layer_inputs[l].vq))
                 for l in range(w.num_layers)]
    # inputs and outputs of E2E_GROUP consecutive layers move in one copy each
    in_groups, host_in, dev_views = layer_groups(per_layer, E2E_GROUP, device)
    out_groups, host_o, out_dev = layer_groups([(o,) for o in rep.outs], E2E_GROUP, device, fill=False)
    desc = [t.contiguous().pin_memory() for t in rep.batch.host]
    dev_in = [(layer,) + dev_views[layer] for layer in range(w.num_layers)]
    host_topk = torch.empty_like(eng.topk_idx, device="cpu").pin_memory() if w.select else None
    h2d = sum(t.numel() * t.element_size() for trip in host_in for t in trip) + sum(
        t.numel() * t.element_size() for t in desc)
    d2h = (host_topk.numel() * 4 if w.select else 0) + sum(o[0].numel() * o[0].element_size() for o in host_o)
    steps = max(3, min(args.steps, 50))
    one = HostStep(eng, dev_in, [v[0] for v in out_dev], None, None, w.impact_layer_index, host_topk=host_topk,
                   batch_host=desc, in_groups=in_groups, out_groups=out_groups, depth=2)
    for _ in range(3):
        one()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    for _ in range(steps):
        one()
    torch.cuda.current_stream().wait_event(one.host_ready())   # the last step's outputs are on the host
    ev1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, device)
    doc = sum(lay.doc_lens)
    return {"value": whole_job_rate(world, doc, steps, ms), "unit": "doc-KV tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps,
            "overlap": f"host copies on copy streams, one copy per {E2E_GROUP} layers each way, two device "
                       "buffer sets alternating between steps, ordered against the kernels by events"}


# ----------------------------------------------------------------------------- selective recompute

RECOMPUTE_CONFIG = "llama3_8b_l32"


def recompute_work(w, n_tok, n_cow):
    """Algorithmic FLOPs and bytes of the recompute, per layer."""
    hk, d, dm = w.num_kv_heads, w.head_dim, w.d_model
    n_out = 2 * hk * d                                         # K and V columns
    gemm_flops = 2 * n_tok * dm * n_out
    gemm_bytes = n_tok * dm * 2 + n_out * dm * 2 + n_tok * n_out * 2
    row_bytes = hk * d * 2                                     # one slot of one page, all KV heads, one tensor
    copy_bytes = 2 * 2 * (n_cow * 16 - n_tok) * row_bytes      # read + write of the non-selected slots, K and V
    return {"gemm_flops": gemm_flops, "gemm_bytes": gemm_bytes, "copy_bytes": copy_bytes}


def run_recompute(args, w, device, do_cpu, ncu=False):
    """Plan once, then every layer's page copy and K/V projection for the
    selection the fused step made on the workload's selecting layer."""
    import serving_prefill_b200 as sp
    from serving_prefill_b200 import Batch, KVPool
    from serving_prefill_b200.engine import PrefillEngine, write_chunks
    from workloads import make_recompute_inputs
    torch.cuda.set_device(device)
    lay = make_layout(w)
    L, li = w.num_layers, w.impact_layer_index
    n_refs = lay.page_ids.numel()
    pool = KVPool(L, lay.num_pages + n_refs, w.num_kv_heads, w.head_dim, dtype=w.torch_dtype, device=device)
    batch = Batch(lay.req_chunk_off, lay.chunk_doc_off, lay.chunk_page_off, lay.page_ids, lay.q_off, device=device)
    eng = PrefillEngine(pool, batch, w.num_q_heads, w.r, dtype=w.torch_dtype, device=device)
    inp = make_layer_inputs(w, lay, li)
    write_chunks(pool, li, [p.to(torch.int32).to(device) for p in lay.chunk_pages],
                 [k.to(device) for k in inp.chunk_k], [v.to(device) for v in inp.chunk_v])
    eng.attend(li, inp.q.to(device), inp.kq.to(device), inp.vq.to(device), with_impact=True)
    eng.select()
    torch.cuda.synchronize()
    k_host = eng.k.cpu().tolist()
    n_sel = sum(k_host)
    plan = torch.empty(sp.rag_recompute_plan_size(batch, eng.k_cap) // 4, dtype=torch.int32, device=device)
    free = torch.arange(lay.num_pages, lay.num_pages + n_refs, dtype=torch.int32, device=device)
    page_out = torch.empty_like(batch.dev[3])
    rin = [make_recompute_inputs(w, lay, layer, rows=n_sel) for layer in range(L)]
    xs = [r.x.to(device) for r in rin]
    wks = [r.w_k.to(device) for r in rin]
    wvs = [r.w_v.to(device) for r in rin]

    def step():
        sp.rag_recompute_plan(batch, eng.topk_idx, eng.k_cap, eng.k, free, page_out, plan, x_by_selection=True)
        for layer in range(L):
            sp.rag_recompute_kv(pool, layer, batch, eng.k_cap, plan, xs[layer], wks[layer], wvs[layer])

    step()
    torch.cuda.synchronize()
    st, counts = sp.rag_recompute_status(plan)
    if st != 0:
        raise RuntimeError(f"recompute status {st}")
    if ncu:   # profiling mode: eager steps only
        for _ in range(args.warmup + args.steps):
            step()
        torch.cuda.synchronize()
        return sp.rag_recompute_status(plan)[0]
    n_tok, n_cow, _ = counts
    s_cap = torch.cuda.Stream()
    s_cap.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s_cap):
        step()
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        g.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(device)
    clocks.start()
    time.sleep(0.2)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    for _ in range(args.steps):
        g.replay()
    ev1.record()
    torch.cuda.synchronize()
    ms = ev0.elapsed_time(ev1)
    clk = clocks.stop()
    # per-kernel device times: the step captured once more with event nodes
    sp.rag_profile_collect()
    sp.rag_profile_enable(True)
    base = sp.rag_launch_count()
    pg = torch.cuda.CUDAGraph()
    with torch.cuda.graph(pg, stream=s_cap):
        step()
    launches = sp.rag_launch_count() - base
    sp.rag_profile_enable(False)
    torch.cuda.synchronize()
    reps = max(3, min(args.steps, 50))
    acc = {}
    for _ in range(reps):
        pg.replay()
        torch.cuda.synchronize()
        for kk, (m_k, c_k) in sp.rag_profile_peek().items():
            a = acc.setdefault(kk, [0.0, 0])
            a[0] += m_k
            a[1] += c_k
    sp.rag_profile_collect()
    del pg, g
    kinds = {kk: v for kk, v in acc.items() if v[1] > 0}
    work = recompute_work(w, n_tok, n_cow)
    peaks = load_peaks()
    tflops_peak = peaks["bf16_tflops_sustained"] if ms > 1000.0 else peaks["bf16_tflops"]
    per_launch = {"rc_gemm": (work["gemm_flops"], work["gemm_bytes"]), "rc_copy": (0, work["copy_bytes"])}
    dom = max((kk for kk in kinds if kk in per_launch), key=lambda kk: kinds[kk][0])
    avg_s = kinds[dom][0] / kinds[dom][1] / 1e3
    flops, nbytes = per_launch[dom]
    if flops:
        ach = flops / avg_s / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": tflops_peak, "unit": "TFLOP/s", "frac": ach / tflops_peak}
    else:
        ach = nbytes / avg_s / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": ach / peaks["hbm_gbs"]}
    roof.update({"kernel": dom, "peak_source": peaks["source"], "avg_launch_us": avg_s * 1e6,
                 "traffic": recorded_traffic("recompute_" + w.name, dom)})
    ms_step = ms / args.steps
    t_roof = max(L * work["gemm_flops"] / (tflops_peak * 1e12),
                 L * (work["gemm_bytes"] + work["copy_bytes"]) / (peaks["hbm_gbs"] * 1e9))
    # end to end through the C ABI: every layer's selected hidden states from pinned host memory,
    # the rewritten page table back to the host
    host_x = [r.x.pin_memory() for r in rin]
    host_pages = torch.empty(page_out.numel(), dtype=torch.int32).pin_memory()
    e2e_steps = max(3, min(args.steps, 20))

    def e2e_step():
        sp.rag_recompute_plan(batch, eng.topk_idx, eng.k_cap, eng.k, free, page_out, plan, x_by_selection=True)
        for layer in range(L):
            xs[layer].copy_(host_x[layer], non_blocking=True)
            sp.rag_recompute_kv(pool, layer, batch, eng.k_cap, plan, xs[layer], wks[layer], wvs[layer])
        host_pages.copy_(page_out, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    ev0.record()
    for _ in range(e2e_steps):
        e2e_step()
    ev1.record()
    torch.cuda.synchronize()
    e2e_ms = ev0.elapsed_time(ev1) / e2e_steps
    entry = {
        "metric": "selected tokens/s through copy-on-write plan + page copy + K/V projection, all layers",
        "value": n_tok / (ms_step / 1e3), "unit": "recomputed tokens/s", "ms_per_step": ms_step,
        "config": {"workload": "recompute_" + w.name, "layers": L, "selected_tokens": n_tok,
                   "private_pages": n_cow, "d_model": w.d_model, "kv_heads": w.num_kv_heads,
                   "selection": "the fused step's top-k on the selecting layer (r = %g)" % w.r,
                   "l2": "per-layer hidden states and weights (%.0f MB in all) exceed L2" %
                         (sum(t.numel() * 2 for t in xs + wks + wvs) / 1e6),
                   "timing": "CUDA graph replay per step"},
        "roofline": roof, "step_roofline": {"t_roof_us": t_roof * 1e6, "t_step_us": ms_step * 1e3,
                                            "frac": t_roof / (ms_step / 1e3)},
        "e2e": {"value": n_tok / (e2e_ms / 1e3), "unit": "recomputed tokens/s",
                "h2d_bytes_per_step": sum(t.numel() * 2 for t in host_x), "d2h_bytes_per_step": page_out.numel() * 4},
        "gpu_launches": int(launches * args.steps), "clocks": clk,
        "kernels": {kk: {"ms_per_step": v[0] / reps, "launches_per_step": v[1] / reps} for kk, v in kinds.items()},
        "work_per_layer": work,
    }
    if do_cpu:
        entry["cpu_baseline"] = recompute_cpu_baseline(w, lay, eng.topk_idx.cpu(), k_host, rin, budget=5.0)
    return entry


def recompute_cpu_baseline(w, lay, topk_idx, k_host, rin, budget):
    """The recompute oracle (plan + copy + projection) on the host cores over a sample of layers."""
    import oracle.prefill as orc
    import oracle.recompute as orc_rc
    sel = [topk_idx[b, :k_host[b]].tolist() for b in range(len(k_host))]
    n_refs = lay.page_ids.numel()
    free = np.arange(lay.num_pages, lay.num_pages + n_refs)
    pk = np.zeros((1, lay.num_pages + n_refs, w.num_kv_heads, 16, w.head_dim), dtype=np.uint16)
    pv = pk.copy()
    t0 = time.perf_counter()
    p = orc_rc.plan(lay.req_chunk_off, lay.chunk_doc_off, lay.chunk_page_off, lay.page_ids, sel, free,
                    x_by_selection=True)
    t_plan = time.perf_counter() - t0
    done, t_layers = 0, 0.0
    while done < w.num_layers and t_layers < budget:
        r = rin[done]
        t0 = time.perf_counter()
        orc_rc.apply(pk, pv, 0, p, orc.to_f64(r.x), orc.to_f64(r.w_k), orc.to_f64(r.w_v))
        t_layers += time.perf_counter() - t0
        done += 1
    t_step = t_plan + t_layers * w.num_layers / done
    return {"value": len(p.x_row) / t_step, "unit": "recomputed tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"plan once, then {done} of {w.num_layers} layers of copy + projection, "
                      f"scaled to all layers; {t_step:.2f} s per step"}


# ----------------------------------------------------------------------------- KV decode into the pool

DECODE_CONFIG = "llama3_8b_l32"


def decode_bits(w, layer):
    """Compression level per part of the cache: 8 bits for the first half of the layers, 4 for the rest."""
    return 8 if layer < w.num_layers // 2 else 4


def run_kv_decode(args, w, device, do_cpu, ncu=False):
    """Every layer of every distinct chunk decoded from its quantized stream into the pool."""
    import serving_prefill_b200 as sp
    from serving_prefill_b200 import KVPool
    from workloads import make_encoded_layer
    torch.cuda.set_device(device)
    lay = make_layout(w)
    L = w.num_layers
    pool = KVPool(L, lay.num_pages, w.num_kv_heads, w.head_dim, dtype=w.torch_dtype, device=device)
    n = list(lay.chunk_len)
    tok_off = torch.tensor(np.cumsum([0] + n), dtype=torch.int32, device=device)
    page_off = torch.tensor(np.cumsum([0] + [len(p) for p in lay.chunk_pages]), dtype=torch.int32, device=device)
    pages = torch.cat(lay.chunk_pages).to(torch.int32).to(device)
    enc = [make_encoded_layer(w, lay, layer, decode_bits(w, layer)) for layer in range(L)]
    dev = [tuple(t.to(device) for t in (e.codes_k, e.codes_v, e.scale_k, e.offset_k, e.scale_v, e.offset_v))
           for e in enc]
    err = torch.zeros(1, dtype=torch.int32, device=device)

    def step(inputs):
        for layer in range(L):
            sp.rag_kv_decode(pool, layer, tok_off, page_off, pages, enc[layer].bits, *inputs[layer], device_err=err)

    step(dev)
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise RuntimeError(f"kv decode device error {int(err.item())}")
    if ncu:   # profiling mode: eager steps only
        for _ in range(args.warmup + args.steps):
            step(dev)
        torch.cuda.synchronize()
        return int(err.item())
    s_cap = torch.cuda.Stream()
    s_cap.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s_cap):
        step(dev)
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        g.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(device)
    clocks.start()
    time.sleep(0.2)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    for _ in range(args.steps):
        g.replay()
    ev1.record()
    torch.cuda.synchronize()
    ms = ev0.elapsed_time(ev1)
    clk = clocks.stop()
    sp.rag_profile_collect()
    sp.rag_profile_enable(True)
    base = sp.rag_launch_count()
    pg = torch.cuda.CUDAGraph()
    with torch.cuda.graph(pg, stream=s_cap):
        step(dev)
    launches = sp.rag_launch_count() - base
    sp.rag_profile_enable(False)
    torch.cuda.synchronize()
    reps = max(3, min(args.steps, 50))
    tot, cnt = 0.0, 0
    for _ in range(reps):
        pg.replay()
        torch.cuda.synchronize()
        m_k, c_k = sp.rag_profile_peek()["kv_decode"]
        tot += m_k
        cnt += c_k
    sp.rag_profile_collect()
    del pg, g
    # algorithmic bytes: codes and scales read, pages written (every slot of every page, K and V)
    n_tok = sum(n)
    n_pages = pages.numel()
    hk, d = w.num_kv_heads, w.head_dim
    per_layer = [2 * n_tok * hk * d * decode_bits(w, l) // 8 + 4 * len(n) * hk * d * 4 +
                 2 * n_pages * hk * 16 * d * 2 for l in range(L)]
    peaks = load_peaks()
    avg_s = tot / cnt / 1e3
    ach = (sum(per_layer) / L) / avg_s / 1e9
    ms_step = ms / args.steps
    t_roof = sum(per_layer) / (peaks["hbm_gbs"] * 1e9)
    roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": ach / peaks["hbm_gbs"],
            "kernel": "kv_decode", "peak_source": peaks["source"], "avg_launch_us": avg_s * 1e6,
            "traffic": recorded_traffic("kv_decode_" + w.name, "kv_decode")}
    # end to end: the compressed stream of every layer from pinned host memory, then decode
    host = [tuple(t.pin_memory() for t in (e.codes_k, e.codes_v, e.scale_k, e.offset_k, e.scale_v, e.offset_v))
            for e in enc]
    e2e_steps = max(3, min(args.steps, 20))

    def e2e_step():
        for layer in range(L):
            for dt, ht in zip(dev[layer], host[layer]):
                dt.copy_(ht, non_blocking=True)
        step(dev)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    ev0.record()
    for _ in range(e2e_steps):
        e2e_step()
    ev1.record()
    torch.cuda.synchronize()
    e2e_ms = ev0.elapsed_time(ev1) / e2e_steps
    h2d = sum(t.numel() * t.element_size() for trip in host for t in trip)
    entry = {
        "metric": "chunk KV tokens/s decoded from quantized streams into the pool, all layers",
        "value": n_tok / (ms_step / 1e3), "unit": "decoded tokens/s (all layers)", "ms_per_step": ms_step,
        "config": {"workload": "kv_decode_" + w.name, "layers": L, "chunks": len(n), "tokens": n_tok,
                   "bits": "8 for layers 0-%d, 4 for layers %d-%d" % (L // 2 - 1, L // 2, L - 1),
                   "l2": "codes of all layers (%.0f MB) and pages (%.0f MB) exceed L2" %
                         (sum(e.codes_k.numel() * 2 for e in enc) / 1e6, pool.k.numel() * 4 / 1e6),
                   "timing": "CUDA graph replay per step"},
        "roofline": roof, "step_roofline": {"t_roof_us": t_roof * 1e6, "t_step_us": ms_step * 1e3,
                                            "frac": t_roof / (ms_step / 1e3)},
        "e2e": {"value": n_tok / (e2e_ms / 1e3), "unit": "decoded tokens/s (all layers)", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": 0},
        "gpu_launches": int(launches * args.steps), "clocks": clk,
        "kernels": {"kv_decode": {"ms_per_step": tot / reps, "launches_per_step": cnt / reps}},
    }
    if do_cpu:
        entry["cpu_baseline"] = kv_decode_cpu_baseline(w, lay, enc, budget=3.0)
    return entry


def kv_decode_cpu_baseline(w, lay, enc, budget):
    """The codec oracle decoding a sample of layers into a host pool."""
    import oracle.codec as codec
    pk = np.zeros((1, lay.num_pages, w.num_kv_heads, 16, w.head_dim), dtype=np.uint16)
    pv = pk.copy()
    done, t = 0, 0.0
    tok0 = np.cumsum([0] + list(lay.chunk_len))
    while done < w.num_layers and t < budget:
        e = enc[done]
        t0 = time.perf_counter()
        for c, pages in enumerate(lay.chunk_pages):
            a, b = tok0[c], tok0[c + 1]
            ch = codec.EncodedChunk(e.bits, e.codes_k[a:b].numpy(), e.codes_v[a:b].numpy(), e.scale_k[c].numpy(),
                                    e.offset_k[c].numpy(), e.scale_v[c].numpy(), e.offset_v[c].numpy())
            codec.decode_into_pool(pk, pv, 0, pages.numpy(), ch, lay.chunk_len[c])
        t += time.perf_counter() - t0
        done += 1
    t_step = t * w.num_layers / done
    return {"value": sum(lay.chunk_len) / t_step, "unit": "decoded tokens/s (all layers)", "cores": blas_threads(),
            "kind": "oracle", "sample": f"{done} of {w.num_layers} layers, scaled to all; {t_step:.2f} s per step"}


# ----------------------------------------------------------------------------- CPU oracle arm

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info] + [1])
    except Exception:
        return os.cpu_count() or 1


def oracle_step(w, lay, layer_inputs, groups, layers=None):
    """The oracle on a sample of KV-head groups of a sample of layers, then top-k.

    A group is one KV head with the G query heads that read it, so a sample
    of n groups is the same problem with n KV heads: its pool, gather and
    attention all shrink in proportion. Layers are independent problems of
    equal size; the selecting layer is always part of the sample.
    """
    import oracle.prefill as orc
    scale = 1.0 / np.sqrt(w.head_dim)
    bits = np.uint16 if w.dtype == "bf16" else np.uint32
    G = w.num_q_heads // w.num_kv_heads
    heads = [g * G + j for g in groups for j in range(G)]
    impact_all = None
    for layer in (range(w.num_layers) if layers is None else layers):
        inp = layer_inputs[layer]
        pk = orc.new_pool(1, lay.num_pages, len(groups), w.head_dim, bits)
        pv = orc.new_pool(1, lay.num_pages, len(groups), w.head_dim, bits)
        for c, pages in enumerate(lay.chunk_pages):
            orc.pool_write(pk, 0, pages.numpy(), orc.to_bits(inp.chunk_k[c][:, groups]))
            orc.pool_write(pv, 0, pages.numpy(), orc.to_bits(inp.chunk_v[c][:, groups]))
        q_all = orc.to_f64(inp.q[:, heads])
        kq_all, vq_all = orc.to_f64(inp.kq[:, groups]), orc.to_f64(inp.vq[:, groups])
        q0 = 0
        imps = []
        for b, cs in enumerate(lay.req_chunks):
            ql = lay.q_lens[b]
            chunks = [(lay.chunk_pages[c].numpy(), lay.chunk_len[c]) for c in cs]
            kd = orc.bits_to_f64(orc.gather(pk, 0, chunks))
            vd = orc.bits_to_f64(orc.gather(pv, 0, chunks))
            n_doc = kd.shape[0]
            kcat = np.concatenate([kd, kq_all[q0:q0 + ql]])
            vcat = np.concatenate([vd, vq_all[q0:q0 + ql]])
            _, _, _, imp, _ = orc.attend_request(q_all[q0:q0 + ql], kcat, vcat, n_doc, scale,
                                                 want_impact=(layer == w.impact_layer_index))
            if imp is not None:
                k = orc.recompute_count(n_doc, w.r)
                orc.select_topk(imp[:n_doc], k)
                imps.append(imp)
            q0 += ql
        if imps:
            impact_all = imps
    return impact_all


def run_reference(args, w, budget_per_step=None):
    lay = make_layout(w)
    layer_inputs = [make_layer_inputs(w, lay, layer) for layer in range(w.num_layers)]
    doc = sum(lay.doc_lens)
    # Calibrate: the sample is a set of layers (the selecting layer first) and
    # of KV-head groups (spread over the heads). Double the layers, then the
    # groups, while one step still fits the per-step budget; the oracle's cost
    # per group depends on how many groups it holds, so it is measured, not
    # extrapolated. When the whole workload fits, all of it is timed.
    budget = budget_per_step or max(0.5, 150.0 / max(1, args.steps + args.warmup))
    L = w.num_layers
    first = w.impact_layer_index if w.impact_layer_index is not None else 0

    def spread(n, total):
        return list(range(0, total, max(1, total // n)))[:n]

    def layer_set(n):
        rest = [x for x in spread(n, L) if x != first]
        return sorted([first] + rest[: n - 1])

    def fits(nl, ng):
        t0 = time.perf_counter()
        oracle_step(w, lay, layer_inputs, spread(ng, w.num_kv_heads), layer_set(nl))
        return time.perf_counter() - t0 <= budget

    nl, ng = 1, 1
    while nl < L and fits(min(2 * nl, L), ng):
        nl = min(2 * nl, L)
    while nl == L and ng < w.num_kv_heads and fits(nl, min(2 * ng, w.num_kv_heads)):
        ng = min(2 * ng, w.num_kv_heads)
    groups, layers = spread(ng, w.num_kv_heads), layer_set(nl)
    for _ in range(args.warmup):
        oracle_step(w, lay, layer_inputs, groups, layers)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(w, lay, layer_inputs, groups, layers)
    dt = time.perf_counter() - t0
    frac = len(groups) / w.num_kv_heads * len(layers) / L
    value = doc * frac * args.steps / dt
    G = w.num_q_heads // w.num_kv_heads
    what = "attention, impact, top-k over all doc tokens" if w.select else "attention (decode step)"
    sample = (f"{len(groups)} of {w.num_kv_heads} KV-head groups ({len(groups) * G} of {w.num_q_heads} query "
              f"heads) of {len(layers)} of {L} layers: pool write, gather, {what}; "
              f"tokens/s scaled by the fraction of (layer, group) pairs timed")
    return value, dt / args.steps, sample


# ----------------------------------------------------------------------------- ranks

def max_over_ranks(ms: float, world: int, device="cpu") -> float:
    """The slowest rank's time: every rank takes part in one MAX reduction."""
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, units_per_rank_step: float, steps: int, ms_max: float) -> float:
    """Units every rank processed in `steps` steps, over the slowest rank's time."""
    return world * units_per_rank_step * steps / (ms_max / 1e3)


# ----------------------------------------------------------------------------- main

def cpu_baseline(w, budget_per_step):
    """The oracle timed on the host cores over a bounded sample of the workload."""
    small = argparse.Namespace(steps=2, warmup=1)
    value, s_per_step, sample = run_reference(small, w, budget_per_step=budget_per_step)
    return {"value": value, "unit": "doc-KV tokens/s" if w.select else "KV tokens/s", "cores": blas_threads(),
            "kind": "oracle", "sample": sample + f"; 2 timed steps of {s_per_step:.2f} s"}


def config_of(w, res, world):
    lay = make_layout(w)
    return {"workload": w.name, "requests": lay.num_requests, "layers": w.num_layers,
            "doc_tokens_per_step": sum(lay.doc_lens), "query_tokens_per_step": lay.total_q,
            "q_heads": w.num_q_heads, "kv_heads": w.num_kv_heads, "head_dim": w.head_dim,
            "r": w.r if w.select else None, "parallelism": f"replicas x{world}",
            "l2": f"inputs rotated over {res['copies']} copies (> L2) between steps",
            "timing": "CUDA graph replay per step"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--impl", default="mine", choices=["mine", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="measure the headline workload only (no per_config block)")
    ap.add_argument("--ncu", action="store_true",
                    help="profiling mode: one input copy, eager launches, W + K steps, no JSON")
    ap.add_argument("--ncu-path", default="step", choices=["step", "recompute", "kv_decode"],
                    help="with --ncu: the fused step, the selective recompute or the KV decode")
    ap.add_argument("--path", default="step", choices=["step", "recompute", "kv_decode"],
                    help="time the selective recompute or the KV decode alone (one JSON line)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    w = get_workload(args.config)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return
        value, s_per_step, sample = run_reference(args, w)
        cores = blas_threads()
        line = {
            "impl": "reference", "metric": METRIC, "value": value, "unit": "doc-KV tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": s_per_step * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "requests": len(make_layout(w).q_lens), "layers": w.num_layers},
            "cpu_baseline": {"value": value, "unit": "doc-KV tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "doc-KV tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line))
        return

    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    device = local
    if args.path != "step" and not args.ncu:
        # one of the further paths alone, timed like its per_config entry
        run = run_recompute if args.path == "recompute" else run_kv_decode
        wp = get_workload(RECOMPUTE_CONFIG if args.path == "recompute" else DECODE_CONFIG)
        entry = run(args, wp, device, not args.no_cpu_baseline)
        entry.update({"n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "higher_is_better": True})
        print(json.dumps(entry))
        return
    if args.ncu and args.ncu_path != "step":
        run = run_recompute if args.ncu_path == "recompute" else run_kv_decode
        st = run(args, w, device, False, ncu=True)
        print(f"ncu mode: {args.warmup + args.steps} eager steps of {args.ncu_path} on {w.name}, status {st}")
        sys.exit(0 if st == 0 else 1)
    if args.ncu:
        torch.cuda.set_device(device)
        lay = make_layout(w)
        rep = Replica(w, lay, [make_layer_inputs(w, lay, layer) for layer in range(w.num_layers)], device)
        for _ in range(args.warmup + args.steps):
            rep.step()
        torch.cuda.synchronize()
        st, bits = rep.engine.device_error()
        print(f"ncu mode: {args.warmup + args.steps} steps of {w.name}, device status {st} ({bits})")
        sys.exit(0 if st == 0 else 1)
    res = run_gpu(args, w, rank, world, device)

    do_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    cpu = cpu_baseline(w, 5.0) if do_cpu else None

    per_config = None
    if world == 1 and not args.no_per_config and args.config == DEFAULT_CONFIG:
        per_config = {}
        for name in PER_CONFIG:
            wc = get_workload(name)
            rc = run_gpu(args, wc, rank, world, device)
            torch.cuda.empty_cache()
            entry = {"value": rc["value"], "unit": "doc-KV tokens/s" if wc.select else "KV tokens/s",
                     "ms_per_step": rc["ms_per_step"], "config": config_of(wc, rc, world),
                     "roofline": rc["roofline"], "step_roofline": rc["step_roofline"],
                     "cpu_baseline": cpu_baseline(wc, 2.0) if do_cpu else None, "e2e": rc["e2e"],
                     "gpu_launches": rc["gpu_launches"], "clocks": rc["clocks"], "kernels": rc["kernels"]}
            per_config[name] = entry
        wr = get_workload(RECOMPUTE_CONFIG)
        per_config["recompute_" + wr.name] = run_recompute(args, wr, device, do_cpu)
        torch.cuda.empty_cache()
        wd = get_workload(DECODE_CONFIG)
        per_config["kv_decode_" + wd.name] = run_kv_decode(args, wd, device, do_cpu)
        torch.cuda.empty_cache()

    if rank == 0:
        line = {
            "metric": METRIC, "value": res["value"], "unit": "doc-KV tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": config_of(w, res, world),
            "roofline": res["roofline"], "step_roofline": res["step_roofline"],
            "cpu_baseline": cpu, "e2e": res["e2e"], "gpu_launches": res["gpu_launches"],
            "clocks": res["clocks"], "kernels": res["kernels"], "kernel_timing": res["kernel_timing"],
        }
        if per_config is not None:
            line["per_config"] = per_config
        print(json.dumps(line))
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
