"""The bench's recorded-traffic lookup: an ncu DRAM figure is reported, scaled
by the touched experts, only while the expert-GEMM sources match the digest
recorded with it; otherwise the bench reports null. Runs without a GPU."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_traffic_reported_only_for_matching_sources(tmp_path, monkeypatch):
    rec = tmp_path / "traffic.json"
    digest = bench.kernel_source_digest()
    rec.write_text(json.dumps({"decode": {"dram_bytes_per_touched_expert": 1000,
                                          "source_digest": digest}}))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(rec))
    assert bench.measured_traffic("decode", 119) == 119000
    assert bench.measured_traffic("prefill", 128) is None  # no record for it
    rec.write_text(json.dumps({"decode": {"dram_bytes_per_touched_expert": 1000,
                                          "source_digest": "0" * 16}}))
    assert bench.measured_traffic("decode", 119) is None  # sources changed since


def test_digest_covers_the_expert_gemm_sources(tmp_path, monkeypatch):
    # the digest changes with either kernel source file
    d0 = bench.kernel_source_digest()
    csrc = tmp_path / "expert_routing_dispatch_router_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in bench.KERNEL_SOURCES:
        with open(os.path.join(ROOT, "expert_routing_dispatch_router_b200", "csrc",
                               name), "rb") as f:
            (csrc / name).write_bytes(f.read())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_source_digest() == d0
    for name in bench.KERNEL_SOURCES:
        p = csrc / name
        original = p.read_bytes()
        p.write_bytes(original + b"\n")
        assert bench.kernel_source_digest() != d0, name
        p.write_bytes(original)


def test_committed_record_is_well_formed():
    with open(bench.TRAFFIC_FILE) as f:
        rec = json.load(f)
    entry = rec["decode"]
    assert entry["dram_bytes_per_touched_expert"] > 0
    assert len(entry["source_digest"]) == 16


def test_headline_workload_traffic_record_is_current():
    # the committed capture of the CTA-pair GEMMs was taken on the current
    # expert-GEMM sources, so the default bench line reports its DRAM traffic
    t = bench.measured_traffic("large_e", 256)
    assert t is not None and 19.3e9 < t < 30e9
