"""The benchmark's host-side bookkeeping on CPU: clock/throttle summary, the
measured-peaks file, the config block, and the rule that a stored DRAM traffic
figure is reported only for the kernel source it was measured on."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402


def _line(sm, mx, hw="Not Active", thermal="Not Active", sw_thermal="Not Active", cap="Not Active"):
    # index, clocks.sm, clocks.max.sm, power.draw, active reasons, then the four reasons
    return f"0, {sm}, {mx}, 700.5, 0x0, {hw}, {thermal}, {sw_thermal}, {cap}"


def test_clock_summary_median_and_reasons():
    c = bench.ClockSampler(0)
    c.lines = [_line(1500, 1965), _line(1600, 1965, cap="Active"), _line(1700, 1965),
               "garbage", ""]
    s = c.summary()
    assert s["sm_mhz"] == 1600.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_summary_reports_slowdowns():
    c = bench.ClockSampler(0)
    c.lines = [_line(900, 1965, hw="Active"), _line(950, 1965, thermal="Active", sw_thermal="Active")]
    s = c.summary()
    assert s["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_clock_summary_without_samples():
    s = bench.ClockSampler(0).summary()
    assert s["sm_mhz"] is None and s["reasons"] == ["unavailable"]


def test_peaks_come_from_the_measured_file():
    p = bench.load_peaks()
    if os.path.exists(bench.PEAKS_FILE):
        assert p["source"] == "measured"
        assert p["bf16"] > p["bf16_sustained"] > 0 and p["hbm"] > 0
    else:
        assert p["source"] == "fallback"


def test_config_names_the_workload_only():
    w = synth.WORKLOADS["long128k"]
    c = bench.config_dict(w, "allgather", 1)
    assert c["workload"] == "long128k" and c["seq_len"] == 131072 and c["rotate"] == "allgather"
    assert "model" not in c
    assert "larger than L2" in c["l2"]


def test_code_digest_ignores_comments_only(tmp_path):
    a = tmp_path / "a.cuh"
    b = tmp_path / "b.cuh"
    c = tmp_path / "c.cuh"
    a.write_text("int f(int x) {  // doubles\n    return 2 * x;\n}\n")
    b.write_text("// a new header comment\nint f(int x) {\n\n    return 2 * x;   // same code\n}\n")
    c.write_text("int f(int x) {\n    return 3 * x;\n}\n")
    assert bench.code_digest(str(a)) == bench.code_digest(str(b))
    assert bench.code_digest(str(a)) != bench.code_digest(str(c))


def test_traffic_reported_only_for_the_measured_source(monkeypatch):
    key = ("long128k", "allgather", "bwd_dkdv")
    rec = bench.MEASURED_TRAFFIC[key]
    path = os.path.join(ROOT, rec["src"])
    current = bench.code_digest(path) == rec["sha256_16"]
    got = bench.measured_traffic(*key)
    assert (got == rec["bytes"]) if current else (got is None)
    # a stale digest turns the figure off; an unmeasured workload or kernel has none
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, key, dict(rec, sha256_16="0" * 16))
    assert bench.measured_traffic(*key) is None
    assert bench.measured_traffic("gqa32k", "ring", "bwd_dkdv") is None
    assert bench.measured_traffic("long128k", "allgather", "fwd") is None
