"""bench.py helpers that need no GPU: the measured-traffic record is reported only
for its own workload and path, and only while the kernel sources match it."""

import json
import os
import shutil

import bench


def test_traffic_record_matches_sources():
    import hashlib

    v = bench.measured_traffic("d4_b1", True)
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "k_mega_d4_b1_dram.json")))
    h = hashlib.sha256()
    for rel in rec["source_files"]:
        h.update(open(os.path.join(bench.ROOT, rel), "rb").read())
    if h.hexdigest() == rec["source_sha256"]:
        assert v == rec["dram_bytes_per_pass"] > 0
    else:  # the kernel changed since the counters were taken: no traffic figure
        assert v is None
    assert bench.measured_traffic("d4_b1", False) is None  # per-phase path: no record
    assert bench.measured_traffic("s8_b16", True) is None  # another workload: no record


def test_traffic_record_dropped_when_kernel_changes(tmp_path, monkeypatch):
    """A record taken on the current sources is reported; editing a source drops it."""
    import hashlib

    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "k_mega_d4_b1_dram.json")))
    os.makedirs(tmp_path / "profiles")
    h = hashlib.sha256()
    for rel in rec["source_files"]:
        os.makedirs(tmp_path / os.path.dirname(rel), exist_ok=True)
        shutil.copy(os.path.join(bench.ROOT, rel), tmp_path / rel)
        h.update(open(tmp_path / rel, "rb").read())
    mine = dict(rec, source_sha256=h.hexdigest(), dram_bytes_per_pass=123456789.0)
    json.dump(mine, open(tmp_path / "profiles" / "k_mega_d4_b1_dram.json", "w"))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("d4_b1", True) == 123456789.0
    with open(tmp_path / rec["source_files"][-1], "a") as f:
        f.write("\n// edited\n")
    assert bench.measured_traffic("d4_b1", True) is None
