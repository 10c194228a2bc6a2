"""The bench's roofline bookkeeping (CPU only).

`bench.py` reports a kernel's DRAM traffic from `profiles/ncu_traffic.json`
only while the kernel's sources hash to the digest recorded with the capture.
These tests pin that machinery: every timed kernel maps to a built source
file, the digest ignores comments and blank lines but not code, and every
record names a known kernel, a plausible byte count and a committed summary.
Whether a record is current is not asserted here: a stale record is reported
as null traffic by the bench itself.
"""

import json
import os
import re

import bench
from serving_prefill_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_every_timed_kernel_maps_to_a_built_source():
    for kernel, src in bench.KERNEL_SOURCE.items():
        assert src in build.SOURCES, f"{kernel}: {src} is not compiled into librag.so"
        assert os.path.exists(os.path.join(build.CSRC, src)), src


def test_digest_ignores_comments_and_blank_lines_only():
    files = {"ptx.cuh": "int a;\n", "common.cuh": "int b;\n", "attn_fwd.cu": "int f() {\n  return 1;\n}\n"}
    base = bench.kernel_sources_digest("attn", files.get)
    commented = dict(files)
    commented["attn_fwd.cu"] = "// a comment\n\nint f() {  // why\n  /* block\n     comment */\n  return 1;\n}\n\n"
    assert bench.kernel_sources_digest("attn", commented.get) == base
    changed = dict(files)
    changed["attn_fwd.cu"] = "int f() {\n  return 2;\n}\n"
    assert bench.kernel_sources_digest("attn", changed.get) != base
    header = dict(files)
    header["ptx.cuh"] = "int a2;\n"
    assert bench.kernel_sources_digest("attn", header.get) != base   # the shared device headers count too


def test_traffic_records_are_well_formed():
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    records = json.load(open(path))
    keys = [k for k in records if not k.startswith("_")]
    assert keys, "no traffic records"
    for key in keys:
        rec = records[key]
        workload, kernel = key.split("/")
        assert kernel in bench.KERNEL_SOURCE, key
        assert workload, key
        assert isinstance(rec["dram_bytes_per_launch"], int) and 0 < rec["dram_bytes_per_launch"] < 200e9, key
        assert re.fullmatch(r"[0-9a-f]{16}", rec["src_digest"]), key
        assert os.path.exists(os.path.join(ROOT, rec["capture"])), f"{key}: {rec['capture']} missing"


def test_recorded_traffic_is_null_for_a_changed_source(monkeypatch):
    # a record whose digest no longer matches is not reported
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    records = json.load(open(path))
    key = next(k for k in records if not k.startswith("_"))
    workload, kernel = key.split("/")
    monkeypatch.setattr(bench, "kernel_sources_digest", lambda k, read=None: "0" * 16)
    assert bench.recorded_traffic(workload, kernel) is None
