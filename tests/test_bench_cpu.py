"""Host logic of bench.py that the reported numbers depend on: the DRAM
traffic figure is reported only for the kernel sources it was measured on,
and the roofline peak falls back to the recipe's figure without the measured
file."""
import json
import os

import bench


def test_traffic_reported_only_while_the_source_hash_matches(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = "0123456789abcdef"
    monkeypatch.setattr(bench, "kernel_source_hash", lambda workload="c1": h)
    (prof / "traffic_c1.json").write_text(json.dumps({"traffic_bytes_per_launch": 1234, "kernel_source_hash": h}))
    assert bench.load_traffic("c1") == 1234
    monkeypatch.setattr(bench, "kernel_source_hash", lambda workload="c1": "fedcba9876543210")
    assert bench.load_traffic("c1") is None          # kernel changed since the capture
    assert bench.load_traffic("c4") is None          # no capture for this workload
    (prof / "traffic_c4.json").write_text("not json")
    assert bench.load_traffic("c4") is None


def test_committed_traffic_records_are_well_formed():
    # each record names the workload's kernel, its bytes and the hash of the
    # sources it was measured on (the bench drops it once they change)
    import re
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    names = [n for n in os.listdir(os.path.join(root, "profiles")) if n.startswith("traffic_") and n.endswith(".json")]
    assert names
    for name in names:
        rec = json.load(open(os.path.join(root, "profiles", name)))
        assert name[len("traffic_"):-len(".json")] in bench.KERNEL_SOURCES, name
        assert rec["traffic_bytes_per_launch"] == rec["dram_bytes_read"] + rec["dram_bytes_write"] > 0, name
        assert re.fullmatch(r"[0-9a-f]{16}", rec["kernel_source_hash"]), name
        assert rec["kernel"] and rec["source"].startswith("ncu "), name


def test_kernel_source_hash_follows_the_sources(tmp_path, monkeypatch):
    csrc = tmp_path / "quantized_expert_matvec_b200" / "csrc"
    csrc.mkdir(parents=True)
    for i, f in enumerate(bench.KERNEL_SOURCES["c1"]):
        (csrc / f).write_text(str(i))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h1 = bench.kernel_source_hash("c1")
    (csrc / "qe_device.cuh").write_text("c")
    assert bench.kernel_source_hash("c1") != h1 and len(h1) == 16


def test_peak_falls_back_without_the_measured_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, kind = bench.measured_peaks()
    assert kind == "fallback" and peaks["hbm_gbs"] == 6650.0
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6554.6}))
    peaks, kind = bench.measured_peaks()
    assert kind == "measured" and peaks["hbm_gbs"] == 6554.6


def test_replica_token_streams_are_disjoint():
    base = 10_000_000
    starts = [bench.rank_token_base(base, r) for r in range(8)]
    # each stream holds fewer than 10^7 tokens, so consecutive bases never overlap
    assert all(b - a >= base for a, b in zip(starts, starts[1:]))
