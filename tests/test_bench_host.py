"""bench.py's host-side rules, on the CPU: the traffic figure is used only for the kernel
sources it was measured on, and the peaks fall back to the stated figures without a
measured-peaks file."""
from __future__ import annotations

import os
import shutil
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


@pytest.fixture
def fake_root(tmp_path, monkeypatch):
    shutil.copytree(os.path.join(ROOT, "int8_quantized_02_b200", "csrc"),
                    tmp_path / "int8_quantized_02_b200" / "csrc")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return tmp_path


def test_traffic_is_used_only_for_the_sources_it_was_taken_on(fake_root):
    h = bench.kernel_source_hash()
    assert len(h) == 16
    (fake_root / "profiles" / "traffic_decode.md").write_text(
        f"# x\n\nkernel_source_hash: {h}\ndram_bytes_per_launch: 67566848\n")
    assert bench.profiled_traffic("decode") == 67566848.0
    assert bench.profiled_traffic("proj175b") is None              # no file
    src = fake_root / "int8_quantized_02_b200" / "csrc" / "decode.cu"
    src.write_bytes(src.read_bytes() + b"\n// changed\n")
    assert bench.kernel_source_hash() != h
    assert bench.profiled_traffic("decode") is None                 # sources changed


def test_peaks_fall_back_without_the_measured_file(fake_root):
    p = bench.measured_peaks()
    assert p["source"] == "fallback" and p["hbm_gbs"] == 6650.0 and p["bf16_tflops"] == 1590.0
    (fake_root / "MEASURED_PEAKS.json").write_text(
        '{"hbm_gbs": 6464.9, "bf16_tflops": 1641.7, "bf16_tflops_sustained": 1368.0}')
    p = bench.measured_peaks()
    assert p["source"] == "measured" and p["hbm_gbs"] == 6464.9
    assert p["bf16_tflops_sustained"] == 1368.0
