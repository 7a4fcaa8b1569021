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



def test_clock_fields_normalise_by_the_sampled_clock():
    # 10 ms at 1500 MHz is 15 Mcycles, 7.63 ms at the 1965 MHz maximum; 1000
    # TFLOP/s on 148 SMs at 1500 MHz is 1000 / (148 * 8192 * 1.5e9 / 1e12) of
    # the tensor peak at that clock
    f = bench.clock_fields(10.0, {"sm_mhz": 1500.0, "samples": 9}, 1000.0, 148)
    assert abs(f["mcycles_per_launch"] - 15.0) < 1e-12
    assert abs(f["ms_at_1965MHz"] - 10.0 * 1500.0 / 1965.0) < 1e-12
    assert abs(f["frac_at_clock"] - 1000.0 / (148 * 8192 * 1.5e9 / 1e12)) < 1e-12
    assert bench.clock_fields(10.0, None, 1000.0, 148) == {"sm_mhz": None}
