"""Clock sampling in the bench: samples are kept only when they fall inside
the timed region, else the two that bracket it; throttle reasons are read
from the reason columns.  A fake sampler process stands in for nvidia-smi."""
import os
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _fake(lines_per_s, first_reason="Not Active", sm=1965):
    period = 1.0 / lines_per_s
    code = ("import sys, time\n"
            "i = 0\n"
            "while True:\n"
            f"    r = {first_reason!r} if i == 0 else 'Not Active'\n"
            f"    print('{sm}, 1965, 500.0, 0x0, Not Active, Not Active, Not Active, ' + r, flush=True)\n"
            "    i += 1\n"
            f"    time.sleep({period})\n")
    return [sys.executable, "-c", code]


def test_samples_inside_long_region():
    s = bench.ClockSampler(0, cmd=_fake(50))
    s.begin()
    time.sleep(0.5)
    c = s.stop()
    assert c["window"] == "inside the timed region"
    assert c["samples"] >= 5 and c["sm_mhz"] == 1965.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == []           # the first sample (power cap) came before begin()


def test_short_region_reports_bracketing_samples():
    s = bench.ClockSampler(0, cmd=_fake(2, sm=1800))
    s.begin()
    c = s.stop()                         # far shorter than the 0.5 s period
    assert c["samples"] == 2 and c["window"].startswith("timed region shorter")
    assert c["sm_mhz"] == 1800.0


def test_reasons_parsed():
    s = bench.ClockSampler(0, cmd=_fake(2, first_reason="Active"))
    s.begin()
    c = s.stop()
    assert "sw_power_cap" in c["reasons"]


def test_missing_sampler():
    s = bench.ClockSampler(0, cmd=["/nonexistent/nvidia-smi"])
    s.begin()
    c = s.stop()
    assert c["sm_mhz"] is None and c["reasons"] == ["nvidia-smi unavailable"]
