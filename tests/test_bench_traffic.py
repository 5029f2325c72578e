"""bench.py's DRAM-traffic records (profiles/traffic.json) hold for the sources
they were captured on: a record is reported only while the hash of its
kernel's sources (its own files plus the shared headers) matches, so a change
to any of those files turns the reported traffic into null until it is
captured again, and a change elsewhere does not (CPU only)."""
import json
import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _tree(tmp_path, monkeypatch):
    csrc = tmp_path / "moe_up_gate_b200" / "csrc"
    shutil.copytree(os.path.join(ROOT, "moe_up_gate_b200", "csrc"), csrc)
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return csrc


def _record(tmp_path, entries):
    with open(tmp_path / "profiles" / "traffic.json", "w") as f:
        json.dump(entries, f)


def test_record_follows_its_sources(tmp_path, monkeypatch):
    csrc = _tree(tmp_path, monkeypatch)
    k = "gemv_batched_kernel"
    _record(tmp_path, {f"wl:{k}": {"dram_bytes_per_launch": 123, "source_hash":
                                   bench.kernel_source_hash(k)}})
    assert bench.recorded_traffic("wl", k) == 123
    assert bench.recorded_traffic("other_workload", k) is None
    for fn, voids in [("q8_matmul.cu", True), ("q8_ptx.cuh", True), ("q8_stream.cuh", True),
                      ("q8_layer.cu", False), ("q8_tc.cu", False)]:
        path = csrc / fn
        orig = path.read_bytes()
        path.write_bytes(orig + b"\n// edited\n")
        assert (bench.recorded_traffic("wl", k) is None) == voids, fn
        path.write_bytes(orig)
        assert bench.recorded_traffic("wl", k) == 123


def test_up_gate_step_covers_both_kernels(tmp_path, monkeypatch):
    csrc = _tree(tmp_path, monkeypatch)
    k = "up_gate_step"
    _record(tmp_path, {f"moe_layer_t256:{k}": {"dram_bytes_per_launch": 7, "source_hash":
                                               bench.kernel_source_hash(k)}})
    assert bench.recorded_traffic("moe_layer_t256", k) == 7
    for fn in ("q8_moe.cu", "q8_tc.cu", "q8_tc.cuh"):
        path = csrc / fn
        orig = path.read_bytes()
        path.write_bytes(orig + b"\n")
        assert bench.recorded_traffic("moe_layer_t256", k) is None, fn
        path.write_bytes(orig)


def test_missing_or_broken_file_reports_nothing(tmp_path, monkeypatch):
    _tree(tmp_path, monkeypatch)
    assert bench.recorded_traffic("wl", "gemv_batched_kernel") is None
    (tmp_path / "profiles" / "traffic.json").write_text("{not json")
    assert bench.recorded_traffic("wl", "gemv_batched_kernel") is None
