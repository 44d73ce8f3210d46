"""Host checks of bench.py's recorded-profile gate: a committed ncu traffic
figure is reported only while the kernel source it was taken on is current."""

import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


@pytest.mark.parametrize("kernel,workload,q", [("decode", "70b", 1), ("verify_tc", "70b", 6)])
def test_recorded_traffic_gate(kernel, workload, q):
    """A record is reported exactly while its source hash is current (a stale
    one reads as null and is skipped here); a current one shows no K/V byte
    read twice."""
    path = os.path.join(ROOT, "profiles", bench.traffic_profile_name(kernel, workload, q))
    with open(path) as f:
        rec = json.load(f)
    traffic = bench.recorded_traffic(kernel, workload, q)
    if rec["kernel_source_sha256_16"] != bench.kernel_hash(kernel):
        assert traffic is None
        pytest.skip(f"{path}: taken on an earlier kernel source")
    assert traffic == rec["dram_bytes_per_launch"]
    assert 0.9 < traffic / rec["algorithmic_bytes_per_launch"] <= 1.0


def test_kernel_hash_ignores_comments(tmp_path, monkeypatch):
    src = tmp_path / "k.cuh"
    src.write_text("int f() { return 1; }  // one\n\n// note\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setitem(bench.KERNEL_SOURCES, "probe", ["k.cuh"])
    h0 = bench.kernel_hash("probe")
    src.write_text("int f() { return 1; }  // changed comment\n// another\n")
    assert bench.kernel_hash("probe") == h0
    src.write_text("int f() { return 2; }\n")
    assert bench.kernel_hash("probe") != h0
