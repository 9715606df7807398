"""Host-side pieces of bench.py (CPU only): the source hash that keys the
committed DRAM counters ignores comments and layout but not code, and a
counter is reported only for the sources it was taken on."""
import json
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_code_only_ignores_comments_and_layout():
    a = "int f(int x) {  // add one\n  return x + 1; /* done */\n}\n"
    b = "int f(int x) {\n    return x + 1;\n}"
    c = "int f(int x) { return x + 2; }"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)


def test_committed_counters_reported_only_for_current_sources():
    """bench.py reports an entry of profiles/traffic.json only while its
    family's code is the one the counters were taken on, and null after a
    kernel edit without a new capture."""
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        entries = json.load(f)
    assert entries
    for key, ent in entries.items():
        family, workload = key.split(":", 1)
        if ent["dram_bytes_per_launch"] is None:
            # a capture that does not cover a whole call records no total
            assert ent.get("note"), key
        else:
            assert ent["dram_bytes_per_launch"] == ent["dram_read_bytes"] + ent["dram_write_bytes"]
        assert os.path.exists(os.path.join(ROOT, ent["capture"])), ent["capture"]
        current = ent["source_hash"] == bench.kernel_source_hash(family)
        expected = ent["dram_bytes_per_launch"] if current else None
        assert bench.traffic_from_profiles(workload, family) == expected, key
    assert bench.traffic_from_profiles("no_such_workload", "tcgen05") is None


def test_alu_peak_from_unit_counts():
    # 148 SMs x 128 fp32 lanes x 2 flops x 1.965 GHz
    assert abs(bench.FP32_ALU_TFLOPS - 74.45) < 0.01
