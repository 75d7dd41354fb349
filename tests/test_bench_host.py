"""bench.py's host-side rules, on the CPU: the peaks fall back to the stated figures without a
measured-peaks file, the prefill peak follows the clock record, and the repeat count and
spread of the repeated timed region."""
from __future__ import annotations

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


@pytest.fixture
def fake_root(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return tmp_path


def test_peaks_fall_back_without_the_measured_file(fake_root):
    p = bench.measured_peaks()
    assert p["source"] == "fallback" and p["hbm_gbs"] == 6650.0 and p["bf16_tflops"] == 1590.0
    (fake_root / "MEASURED_PEAKS.json").write_text(
        '{"hbm_gbs": 6464.9, "bf16_tflops": 1641.7, "bf16_tflops_sustained": 1368.0}')
    p = bench.measured_peaks()
    assert p["source"] == "measured" and p["hbm_gbs"] == 6464.9
    assert p["bf16_tflops_sustained"] == 1368.0


def test_repeat_count():
    assert bench.repeat_count(0.001, 1.0) == 200           # capped
    assert bench.repeat_count(0.01, 1.0) == 100
    assert bench.repeat_count(0.3, 1.0) == 4               # ceil(1 / 0.3)
    assert bench.repeat_count(2.0, 1.0) == 3               # at least three
    assert bench.repeat_count(0.0, 1.0) == 200
    assert bench.repeat_count(0.1, 1.0, lo=3, hi=5) == 5


def test_spread():
    s = bench.spread([5.0, 1.0, 3.0, 2.0, 4.0])
    assert s["n"] == 5 and s["median"] == 3.0 and s["min"] == 1.0 and s["max"] == 5.0
    assert s["p10"] == 1.0 and s["p90"] == 5.0
    s = bench.spread([float(i) for i in range(101)])
    assert s["p10"] == 10.0 and s["p90"] == 90.0 and s["median"] == 50.0


def test_int8_peak_follows_the_clock_record():
    assert bench.int8_peak_kind({"sm_mhz": 1780, "sm_max_mhz": 1965,
                                 "reasons": ["sw_power_cap"]}) == ("bf16_tflops_sustained", True)
    # clocks held well below the maximum with no reason recorded: not the burst regime either
    assert bench.int8_peak_kind({"sm_mhz": 1500, "sm_max_mhz": 1965, "reasons": []})[0] == \
        "bf16_tflops_sustained"
    assert bench.int8_peak_kind({"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []}) == \
        ("bf16_tflops", False)
    # no NVML: no evidence of a cap
    assert bench.int8_peak_kind({"sm_mhz": None, "sm_max_mhz": None, "reasons": []}) == \
        ("bf16_tflops", False)
