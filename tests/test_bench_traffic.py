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
    ent = t["main_branch"]
    src = os.path.join(ROOT, "block_sparse_long_branch_b200", "csrc", ent["source"])
    with open(src, "rb") as f:
        current = hashlib.sha256(f.read()).hexdigest()[:16] == ent["source_sha"]
    got = bench.traffic_for("main_branch", t["workload"])
    assert got == (ent["bytes_per_launch"] if current else None)
    assert bench.traffic_for("main_branch", "prefill_1m") is None
    assert bench.traffic_for("main_branch", None) is None
    assert bench.traffic_for("decode_index", t["workload"]) is None
