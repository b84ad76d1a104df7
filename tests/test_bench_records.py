"""bench.py reports a committed ncu traffic record only for the kernel source and
the workload it was captured on (profiles/round_attn_traffic.json,
profiles/kv_append_traffic.json)."""
import json
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _record(name):
    with open(os.path.join(ROOT, "profiles", name)) as f:
        return json.load(f)


def test_attention_traffic_record_is_keyed_to_source_and_workload(monkeypatch):
    rec = _record("round_attn_traffic.json")
    key = rec["workload_key"]
    assert key in bench.WORKLOADS
    same_source = rec["kernel_source_sha256"] == bench._kernel_source_hash()
    assert bench._measured_traffic(key) == (rec["dram_bytes_per_launch"] if same_source else None)
    for other in bench.WORKLOADS:
        if other != key:
            assert bench._measured_traffic(other) is None, other
    monkeypatch.setattr(bench, "_kernel_source_hash", lambda: "another source")
    assert bench._measured_traffic(key) is None


def test_append_traffic_record_is_keyed_to_source_and_workload(monkeypatch):
    rec = _record("kv_append_traffic.json")
    key = rec["workload_key"]
    assert key in bench.WORKLOADS
    same_source = rec["kernel_source_sha256"] == bench._source_hash(["wave_device.cu"])
    got = bench._measured_append_traffic(key)
    if same_source:
        assert got == {k: rec[k] for k in ("dram_read_bytes", "dram_write_bytes", "duration_ns")}
    else:
        assert got is None
    for other in bench.WORKLOADS:
        if other != key:
            assert bench._measured_append_traffic(other) is None, other
    monkeypatch.setattr(bench, "_source_hash", lambda names: "another source")
    assert bench._measured_append_traffic(key) is None
