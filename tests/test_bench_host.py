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


def test_every_workload_parses_with_its_metric(monkeypatch):
    cases = {
        ("--workload", "body8b"): ("us/pass", bench.HEADLINE_METRIC),
        ("--workload", "layer8b"): ("us/layer", None),
        ("--workload", "body27b", "--batch", "4"): ("us/pass", None),
        ("--workload", "pq2_body8b"): ("us/pass", None),
        ("--workload", "sweep", "--matrix", "down", "--batch", "64"): ("us/product", None),
        ("--workload", "format", "--case", "base3"): ("us/call", None),
    }
    for argv, (unit, metric) in cases.items():
        a = bench.parse(list(argv))
        m, u = bench.metric_of(a)
        assert u == unit
        if metric:
            assert m == metric
        assert bench.workload_text(a)
    # the headline metric is BASELINE's only at the default workload and batch 1
    assert bench.metric_of(bench.parse(["--batch", "4"]))[0] != bench.HEADLINE_METRIC
    assert bench.parse([]).steps == 200 and bench.parse(["--workload", "format"]).steps == 20


def test_oracle_sample_is_layer_zero_and_scales_to_a_step():
    """The CPU baseline samples the seven matrices of layer 0 and scales by
    weight count: x36 for the 8B pass, x64 for the 27B one, x1 for one layer
    and for the sweep's single product."""
    for argv, scale in ((["--workload", "body8b"], 36), (["--workload", "body27b"], 64),
                        (["--workload", "layer8b"], 1), (["--workload", "sweep", "--matrix", "gate"], 1)):
        a = bench.parse(argv)
        units, step_w = bench.oracle_units(a)
        assert len(units) == (1 if a.workload == "sweep" else 7)
        assert step_w == scale * sum(w for _, w, _ in units)
    assert bench.oracle_units(bench.parse(["--workload", "format"])) == ([], 0)


def test_reference_arm_times_what_it_runs(monkeypatch, capsys):
    """ms_per_step is the measured time of the sampled matrix each step ran;
    value scales the per-matrix means to a whole step by weight count."""
    import json
    import time as _t
    units = [("a", 10, lambda: (lambda: _t.sleep(0.02))), ("b", 30, lambda: (lambda: _t.sleep(0.04)))]
    monkeypatch.setattr(bench, "oracle_units", lambda a: (units, 80))
    a = bench.parse(["--impl", "reference", "--steps", "4", "--warmup", "1"])
    bench.run_reference(a)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["steps"] == 4
    # steps ran units b, a, b, a (warm-up took a): mean step 30 ms
    assert 25 < line["ms_per_step"] < 60
    # value = (mean a + mean b) * 80 / 40 = (20 + 40 ms) * 2 = 120 ms
    assert 100e3 < line["value"] < 180e3
    assert line["e2e"]["value"] == line["value"] and line["cpu_baseline"]["kind"] == "oracle"


def test_weight_and_flop_counts():
    # the 8B gate: 12288 x 4096, k = 8, r = 8 (layout v1 payload, before padding)
    assert bench.weight_bytes(12288, 4096, 8, 8) == 12288 * 4096 // 4 + 12288 * 32 * 8 + 12288 * 32 * 4 + \
        12288 * 4 + 8 * 4096 // 8 + 16
    assert bench.pq2_bytes(12288, 4096) == 12288 * 32 * 34
    assert bench.product_flops(12288, 4096, 8, 16, 64) == 2 * 64 * 12288 * 4096 + 2 * 64 * 12288 * 32 * 8 + \
        2 * 64 * 16 * (12288 + 4096)
