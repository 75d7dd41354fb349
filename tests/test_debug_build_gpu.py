"""The debug build (libllmint8_debug.so, compiled with LLMINT8_DEBUG): its device-side bounds
checks (outlier column index < K, listed count <= capacity, stores inside the output) hold on
the small and odd shapes of the parity tests, whose results stay those of the oracle.  A
failed check would show as LLMINT8_ERR_DEVICE_CHECK in the device status, which those tests
require to be LLMINT8_OK."""
from __future__ import annotations

import os
import subprocess
import sys

import pytest

from int8_quantized_02_b200 import build as build_mod

pytestmark = pytest.mark.gpu

SELECT = " or ".join([
    "test_quantize_rows_bitexact", "test_linear_matches_oracle",
    "test_linear_zero_and_outlier_only_rows", "test_decode_path_matches_oracle",
    "test_decode_path_planted_rows", "test_gemm_path_small_M",
])


def test_parity_cases_pass_under_the_debug_build():
    build_mod.build(debug=True)
    env = dict(os.environ, LLMINT8_DEBUG="1")
    probe = subprocess.run(
        [sys.executable, "-c",
         "from int8_quantized_02_b200 import llmint8 as L; "
         "assert L.build_flags() & 1; print(L.library_path())"],
        cwd=build_mod.ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert probe.returncode == 0, probe.stderr[-2000:]
    assert probe.stdout.strip().endswith("libllmint8_debug.so")
    run = subprocess.run(
        [sys.executable, "-m", "pytest", os.path.join("tests", "test_parity_gpu.py"), "-m",
         "gpu", "-q", "-x", "-p", "no:cacheprovider", "-k", SELECT],
        cwd=build_mod.ROOT, env=env, capture_output=True, text=True, timeout=1800)
    assert run.returncode == 0, run.stdout[-4000:] + run.stderr[-2000:]
    assert " passed" in run.stdout
