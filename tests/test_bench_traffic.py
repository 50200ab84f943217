"""bench.py's `roofline.traffic`: the DRAM bytes of a stage come from the
committed ncu summary only while the kernel sources it names are unchanged
(their digest is stored beside the bytes); any change, a missing entry or a
malformed file gives null."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _tree(tmp_path, body=b"__global__ void k() {}\n"):
    src = tmp_path / "k.cu"
    src.write_bytes(body)
    (tmp_path / "profiles").mkdir()
    return src


def _write(tmp_path, entry):
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"wl": {"bwd": entry}}))


def test_bytes_returned_while_the_sources_match(tmp_path, monkeypatch):
    _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    _write(tmp_path, {"bytes": 1234, "sources": ["k.cu"], "digest": bench.source_digest(["k.cu"])})
    assert bench.measured_traffic("wl", "bwd") == 1234


def test_null_once_a_source_changes(tmp_path, monkeypatch):
    src = _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    _write(tmp_path, {"bytes": 1234, "sources": ["k.cu"], "digest": bench.source_digest(["k.cu"])})
    src.write_bytes(b"__global__ void k() { /* changed */ }\n")
    assert bench.measured_traffic("wl", "bwd") is None


def test_null_for_missing_entries_and_bad_files(tmp_path, monkeypatch):
    _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("wl", "bwd") is None            # no file
    _write(tmp_path, {"bytes": 1, "sources": ["k.cu"], "digest": bench.source_digest(["k.cu"])})
    assert bench.measured_traffic("wl", "fwd") is None            # no such stage
    assert bench.measured_traffic("other", "bwd") is None         # no such workload
    _write(tmp_path, {"bytes": 1, "sources": ["gone.cu"], "digest": "0"})
    assert bench.measured_traffic("wl", "bwd") is None            # source missing
    (tmp_path / "profiles" / "traffic.json").write_text("{not json")
    assert bench.measured_traffic("wl", "bwd") is None            # malformed


def test_committed_summary_names_existing_sources():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        data = json.load(f)
    for wl, stages in data.items():
        if wl.startswith("_"):
            continue
        for stage, e in stages.items():
            assert e["bytes"] > 0
            for s in e["sources"]:
                assert os.path.exists(os.path.join(ROOT, s)), (wl, stage, s)
