"""bench.py helpers that need no GPU: the measured-traffic record is reported only
for its own workload and path, and only while the kernel sources match it."""

import json
import os
import shutil

import bench


def test_traffic_record_matches_sources():
    v = bench.measured_traffic("d4_b1", True)
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "k_mega_d4_b1_dram.json")))
    assert v == rec["dram_bytes_per_pass"] > 0
    assert bench.measured_traffic("d4_b1", False) is None  # per-phase path: no record
    assert bench.measured_traffic("s8_b16", True) is None  # another workload: no record


def test_traffic_record_dropped_when_kernel_changes(tmp_path, monkeypatch):
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "k_mega_d4_b1_dram.json")))
    os.makedirs(tmp_path / "profiles")
    shutil.copy(os.path.join(bench.ROOT, "profiles", "k_mega_d4_b1_dram.json"), tmp_path / "profiles")
    for rel in rec["source_files"]:
        os.makedirs(tmp_path / os.path.dirname(rel), exist_ok=True)
        shutil.copy(os.path.join(bench.ROOT, rel), tmp_path / rel)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("d4_b1", True) == rec["dram_bytes_per_pass"]
    with open(tmp_path / rec["source_files"][-1], "a") as f:
        f.write("\n// edited\n")
    assert bench.measured_traffic("d4_b1", True) is None
