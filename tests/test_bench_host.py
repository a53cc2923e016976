"""Host-side logic of bench.py that needs no GPU: the roofline traffic figure comes from the
committed ncu summary only while the library sources are the ones those counters were taken on."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402


def test_traffic_summary_is_parseable():
    fields = {}
    with open(bench.TRAFFIC_PROFILE) as fh:
        for line in fh:
            if ":" in line:
                k, v = line.split(":", 1)
                fields[k.strip()] = v.strip()
    assert int(fields["traffic_bytes_per_launch"]) > 0
    assert len(fields["sources_sha256"]) == 64


def test_traffic_is_null_once_sources_change(monkeypatch):
    monkeypatch.setattr(bench, "library_sources_sha256", lambda: "0" * 64)
    assert bench.measured_traffic() is None


def test_traffic_follows_the_recorded_hash(monkeypatch, tmp_path):
    p = tmp_path / "summary.md"
    p.write_text("text: x\ntraffic_bytes_per_launch: 1234\nsources_sha256: " + "a" * 64 + "\n")
    monkeypatch.setattr(bench, "TRAFFIC_PROFILE", str(p))
    monkeypatch.setattr(bench, "library_sources_sha256", lambda: "a" * 64)
    assert bench.measured_traffic() == 1234
