"""bench.py's bookkeeping, on CPU: every workload names its dominant kernel,
every kernel named has its sources listed, and a captured DRAM figure is
reported only while the sources it was taken at are unchanged."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_every_workload_names_a_dominant_kernel_with_sources():
    assert set(bench.DOMINANT) == set(bench.W.WORKLOADS)
    for kernel in bench.DOMINANT.values():
        assert kernel in bench.KERNEL_SOURCES
        for f in bench.KERNEL_SOURCES[kernel]:
            assert os.path.exists(os.path.join(ROOT, "adapter_lora_serving_b200", "csrc", f)), f


def test_traffic_entries_match_their_kernels_and_captures():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as fh:
        table = json.load(fh)
    for name, rec in table.items():
        assert rec["kernel"] == bench.DOMINANT[name], name
        assert os.path.exists(os.path.join(ROOT, rec["capture"])), rec["capture"]
        assert rec["dram_bytes_per_launch"] > 0


def test_traffic_is_dropped_when_the_sources_change(monkeypatch):
    name = next(iter(json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))))
    kernel = bench.DOMINANT[name]
    real = bench.source_digest
    monkeypatch.setattr(bench, "source_digest", lambda k: "0" * 16 if k == kernel else real(k))
    traffic, named = bench.measured_traffic(name)
    assert traffic is None and named == kernel
