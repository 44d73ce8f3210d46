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


def _cfg():
    from paged_kv_cache_381_b200 import workloads as wl
    return wl.DecodeConfig("bytes", "bf16", 3, 4, 2, 64, 16, "fixed", fixed_lengths=(10, 20, 40))


def test_algorithmic_bytes_hand_example():
    """Contexts 10, 20, 40 with 16-token partitions and blocks; 4 query / 2 kv
    heads, head_dim 64, bf16.  By hand: K/V 70 tokens x 2 x 2 heads x 64 x 2 B
    = 35840; q 3 x 4 x 64 x 2 = 1536; the one single-partition sequence's rows
    4 x 64 x 2 = 512; partials of 2 + 3 partitions x 4 heads x (64 + 2) x 4 B
    = 5280; table entries (1 + 2 + 3) blocks x 2 kv heads x 4 B = 48."""
    import numpy as np
    cfg, lens = _cfg(), np.array([10, 20, 40])
    assert bench.kv_bytes(cfg, lens) == 35840
    assert bench.decode_kernel_bytes(cfg, lens, 16) == 35840 + 1536 + 512 + 5280 + 48
    # merged in the kernel: every final row written, partials written and read back
    assert bench.decode_kernel_bytes(cfg, lens, 16, fused=True) == 35840 + 1536 + 1536 + 2 * 5280 + 48
    # one partition for everything: no partials
    assert bench.decode_kernel_bytes(cfg, lens, 64) == 35840 + 1536 + 1536 + 48


def test_verify_bytes_and_flops_hand_example():
    """Two query rows per sequence: q and rows double, partials double; flops
    4 x D x Hq x (visible positions) with 9 + 10, 19 + 20, 39 + 40 visible."""
    import numpy as np
    cfg, lens = _cfg(), np.array([10, 20, 40])
    assert bench.verify_kernel_bytes(cfg, lens, 16, 2) == 35840 + 3072 + 1024 + 10560 + 48
    assert bench.verify_flops(cfg, lens, 2) == 4 * 64 * 4 * (19 + 39 + 79)
    assert bench.verify_kernel_bytes(cfg, lens, 16, 1) == bench.decode_kernel_bytes(cfg, lens, 16)


def test_reference_arm_reports_the_native_config(tmp_path):
    """The reference arm prints the native arm's config object (same keys and
    values for the same workload), so the two lines describe one workload."""
    import json
    import subprocess
    import sys
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "tiny", "--steps", "1", "--warmup", "0"], capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr
    line = json.loads(res.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    cfg = bench.wl.CONFIGS["tiny"]
    lens = bench.wl.context_lengths(cfg, bench.wl.rng(0))

    class A:
        workload, math, merge, partition_size = "tiny", "auto", "kernel", 0
    assert line["config"] == bench.workload_config(A, cfg, lens, cfg.partition_size, 1)
    assert line["config"]["kv_bytes_per_step"] == bench.kv_bytes(cfg, lens)
    assert set(line["e2e"]) >= {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"}
