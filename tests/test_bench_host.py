"""Host-side logic of bench.py that needs no GPU: the roofline traffic figure comes from the
committed capture record only while the library sources are the ones those counters were taken on."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402


def test_traffic_record_is_parseable():
    import json
    with open(bench.TRAFFIC_DATA) as fh:
        rec = json.load(fh)
    assert int(rec["traffic_bytes_per_launch"]) == int(rec["dram_bytes_read"]) + int(rec["dram_bytes_write"]) > 0
    assert len(rec["sources_sha256"]) == 64 and "--clock-control none" in rec["command"]


def test_traffic_is_null_once_sources_change(monkeypatch):
    monkeypatch.setattr(bench, "library_sources_sha256", lambda: "0" * 64)
    assert bench.measured_traffic() is None


def test_traffic_follows_the_recorded_hash(monkeypatch, tmp_path):
    p = tmp_path / "record.json"
    p.write_text('{"traffic_bytes_per_launch": 1234, "sources_sha256": "' + "a" * 64 + '"}')
    monkeypatch.setattr(bench, "TRAFFIC_DATA", str(p))
    monkeypatch.setattr(bench, "library_sources_sha256", lambda: "a" * 64)
    assert bench.measured_traffic() == 1234


def _clock_line(t, sm, pcap="Not Active", hw="Not Active"):
    return f"{t}, 0, {sm}, 1965, 600.5, 0x0, {hw}, Not Active, Not Active, {pcap}\n"


def test_clock_samples_inside_the_timed_region():
    import datetime
    lines = [_clock_line("2026/12/02 10:00:00.000", 1200), _clock_line("2026/12/02 10:00:00.050", 1800, "Active"),
             _clock_line("2026/12/02 10:00:00.100", 1700), _clock_line("2026/12/02 10:00:00.150", 900, hw="Active")]
    t0 = datetime.datetime(2026, 12, 2, 10, 0, 0, 40000)
    t1 = datetime.datetime(2026, 12, 2, 10, 0, 0, 120000)
    s = bench.summarize_clock_samples(lines, t0, t1)
    assert s["samples"] == 2 and s["sm_mhz"] == 1750 and s["reasons"] == ["sw_power_cap"]
    assert s["window"] == "timed region"


def test_clock_samples_adjacent_to_a_short_region():
    import datetime
    lines = [_clock_line("2026/12/02 10:00:00.000", 1500), _clock_line("2026/12/02 10:00:00.050", 1600),
             _clock_line("2026/12/02 10:00:00.100", 1700, hw="Active")]
    t0 = datetime.datetime(2026, 12, 2, 10, 0, 0, 60000)
    t1 = datetime.datetime(2026, 12, 2, 10, 0, 0, 80000)
    s = bench.summarize_clock_samples(lines, t0, t1)
    assert s["samples"] == 2 and s["sm_mhz"] == 1650 and s["reasons"] == ["hw_slowdown"]
    assert s["window"].startswith("adjacent")
    assert bench.summarize_clock_samples(["garbage\n"], t0, t1)["reasons"] == ["no samples"]


def test_traffic_hash_ignores_comments_only():
    code = "int a = 1;  // one\n\n// a note\nint b = 2;\n"
    assert bench._code_only(code) == bench._code_only("int a = 1;  // changed\nint b = 2;   \n")
    assert bench._code_only(code) != bench._code_only("int a = 1;\nint b = 3;\n")
