"""Host logic of bench.py that decides what its JSON line reports: the DRAM
traffic of the fused GEMM is reported only while the kernel sources are the
ones the counters were taken on (null once they change, or when the record
is missing), and the clock summary is the median of the samples taken."""
import hashlib
import json
import os

import bench


def _record(root, sources, content):
    os.makedirs(os.path.join(root, "profiles"), exist_ok=True)
    h = hashlib.sha256()
    for rel, text in zip(sources, content):
        path = os.path.join(root, rel)
        os.makedirs(os.path.dirname(path), exist_ok=True)
        with open(path, "w") as f:
            f.write(text)
        h.update(text.encode())
    rec = {"source_sha256_16": h.hexdigest()[:16], "sources": sources,
           "dram_bytes_read": 1000, "dram_bytes_write": 234}
    with open(os.path.join(root, "profiles", "traffic_gemm_pair_fused_gdn_8192x24704x5120.json"), "w") as f:
        json.dump(rec, f)


def test_traffic_reported_only_for_the_profiled_sources(tmp_path, monkeypatch):
    root = str(tmp_path)
    monkeypatch.setattr(bench, "ROOT", root)
    assert bench.gemm_traffic() is None                      # no record
    srcs = ["csrc/a.cu", "csrc/b.cuh"]
    _record(root, srcs, ["kernel A\n", "header B\n"])
    assert bench.gemm_traffic() == 1234                      # sources as profiled
    with open(os.path.join(root, "csrc/b.cuh"), "a") as f:
        f.write("// changed\n")
    assert bench.gemm_traffic() is None                      # kernel changed since
    os.remove(os.path.join(root, "csrc/b.cuh"))
    assert bench.gemm_traffic() is None                      # source missing


def test_committed_traffic_record_is_well_formed():
    # the record in the repository names existing sources and a full launch's bytes
    path = os.path.join(bench.ROOT, "profiles", "traffic_gemm_pair_fused_gdn_8192x24704x5120.json")
    with open(path) as f:
        rec = json.load(f)
    for src in rec["sources"]:
        assert os.path.exists(os.path.join(bench.ROOT, src)), src
    assert rec["dram_bytes_read"] > 0 and rec["dram_bytes_write"] > 0
    assert "--clock-control none" in rec["command"]


def test_clock_summary_is_the_median_of_the_samples():
    c = bench.ClockSampler.__new__(bench.ClockSampler)
    c.samples, c.reasons, c.max_mhz = [1965, 1800, 1950, 1965, 1900], {"sw_power_cap"}, 1965
    s = c.summary()
    assert s == {"sm_mhz": 1950.0, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"], "samples": 5}
    c.samples = []
    assert c.summary()["sm_mhz"] is None and c.summary()["samples"] == 0
