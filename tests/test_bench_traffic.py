"""bench.py's DRAM-traffic lookup: a committed ncu figure is reported only for
the workload it was captured on, and only while the kernel source is unchanged."""
import hashlib
import json
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _table():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        return json.load(f)


def test_traffic_only_for_the_captured_workload():
    t = _table()
    for kernel in ("index_select", "main_branch"):
        ent = t[kernel]
        src = os.path.join(ROOT, "block_sparse_long_branch_b200", "csrc", ent["source"])
        with open(src, "rb") as f:
            current = hashlib.sha256(f.read()).hexdigest()[:16] == ent["source_sha"]
        assert ent["bytes_per_phase"] == ent["read"] + ent["write"]
        got = bench.traffic_for(kernel, ent["workload"])
        assert got == (ent["bytes_per_phase"] if current else None)
        assert bench.traffic_for(kernel, "prefill_tiny_other") is None
        assert bench.traffic_for(kernel, None) is None
    assert bench.traffic_for("decode_index", t["index_select"]["workload"]) is None
