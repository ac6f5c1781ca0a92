"""bench.py reports a kernel's DRAM traffic from a committed ncu record only
while the kernel's source file is unchanged since the capture."""
import json
import os

import pytest

pytest.importorskip("numpy")


def _tree(tmp_path, src, rec):  # a repository layout with one kernel source
    csrc = tmp_path / "mxfp4_routed_expert_v4moe_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text(src)
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))


def test_traffic_follows_the_kernel_source(tmp_path, monkeypatch):
    import bench
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    _tree(tmp_path, "kernel v1", {})
    h1 = bench.source_hash("k.cu")
    rec = {"kern@wl": {"file": "k.cu", "hash": h1, "bytes_per_launch": 123}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    assert bench.recorded_traffic("kern", "wl") == 123
    assert bench.recorded_traffic("kern", "other_workload") is None
    (tmp_path / "mxfp4_routed_expert_v4moe_b200" / "csrc" / "k.cu").write_text("kernel v2")
    assert bench.recorded_traffic("kern", "wl") is None  # the kernel changed since the capture


def test_committed_records_name_existing_sources():
    import bench
    d = json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))
    for key, e in d.items():
        assert "@" in key and e["bytes_per_launch"] > 0
        assert bench.source_hash(e["file"]) is not None, e["file"]
