"""Host logic of bench.py that needs no GPU: the clock record keeps only the
samples taken inside the timed window, and the step default depends on the
arm."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _sampler(rows):
    c = bench.ClockSampler(0)
    c.rows = list(rows)
    c.source = "nvml"
    return c


def test_clock_summary_keeps_the_window():
    rows = [(0.0, 345.0, 1965.0, []),                # idle, before the window
            (1.0, 1965.0, 1965.0, []),
            (1.5, 1900.0, 1965.0, ["sw_power_cap"]),
            (2.0, 1950.0, 1965.0, []),
            (3.0, 400.0, 1965.0, ["hw_slowdown"])]  # after the window
    s = _sampler(rows).summary(0.9, 2.1)
    assert s["samples"] == 3
    assert s["sm_mhz"] == 1950.0 and s["sm_min_mhz"] == 1900.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]
    assert s["window_ms"] == 1000.0


def test_clock_summary_without_samples_says_so():
    s = _sampler([(0.0, 1965.0, 1965.0, [])]).summary(1.0, 2.0)
    assert s["samples"] == 0 and s["reasons"] == ["unsampled"] and s["sm_mhz"] is None


def test_step_default_per_arm(monkeypatch):
    monkeypatch.setattr(sys, "argv", ["bench.py"])
    assert bench.parse().steps == 200
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference"])
    assert bench.parse().steps == 20
    monkeypatch.setattr(sys, "argv", ["bench.py", "--steps", "7"])
    assert bench.parse().steps == 7
