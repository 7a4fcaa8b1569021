"""Host-side pieces of bench.py that need no GPU: the DRAM-traffic record is
reported only while the kernel sources hash to the value it was captured
with, and null (None) once they differ."""
import json

import bench


def test_traffic_is_reported_only_for_the_captured_sources(tmp_path, monkeypatch):
    rec = {"csrc_sha256": bench.kernel_sources_sha256(),
           "forward": {"dram_read_bytes": 10, "dram_write_bytes": 2},
           "backward": {"dram_read_bytes": 30, "dram_write_bytes": 4}}
    f = tmp_path / "traffic.json"
    f.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.measured_traffic() == (12, 34)
    rec["csrc_sha256"] = "0" * 64                       # sources changed since the capture
    f.write_text(json.dumps(rec))
    assert bench.measured_traffic() == (None, None)
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "missing.json"))
    assert bench.measured_traffic() == (None, None)

