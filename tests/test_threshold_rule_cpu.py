"""The outlier test |x| >= t on fp16 x, as the kernels take it: packed fp16 compares of |x|
against the smallest fp16 at or above t.  Checked here on the CPU for every fp16 bit pattern
(NaN and infinities included) against the plain comparison in float64, for thresholds that
are fp16 values, lie between them, are zero or negative, or lie past the fp16 range."""
from __future__ import annotations

import numpy as np
import pytest


def smallest_fp16_at_or_above(t: float) -> float:
    """The least fp16 value >= t, as a float64 (+inf when t is above the largest fp16)."""
    if np.isinf(t):
        return t
    with np.errstate(over="ignore"):
        h = np.float16(t)                   # round to nearest (may round down)
        if np.float64(h) < t:
            h = np.nextafter(h, np.float16(np.inf))   # past 65504: +inf
    return float(h)


ALL_FP16 = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16).view(np.float16)

THRESHOLDS = [6.0, 6.001, 5.999, 6.00390625, 2.5, 1.0 / 3.0, 1e-8, 6.0e-8, 0.0, -0.0, -1.0,
              65504.0, 65504.5, 65520.0, 70000.0, 1e30, float("inf"), -float("inf")]


@pytest.mark.parametrize("t", THRESHOLDS)
def test_rounded_threshold_flags_exactly_the_plain_comparison(t):
    a = np.abs(ALL_FP16.astype(np.float64))          # |x|, exact; NaN stays NaN
    with np.errstate(invalid="ignore"):
        plain = a >= t
        t16 = smallest_fp16_at_or_above(t)
        assert np.float64(np.float16(t16)) == t16        # an fp16 value (or an infinity)
        rounded = np.abs(ALL_FP16) >= np.float16(t16)
    assert np.array_equal(plain, rounded), f"t = {t!r}"
    # NaN is never an outlier; infinities are, for every finite threshold
    assert not plain[np.isnan(ALL_FP16)].any()
    if np.isfinite(t):
        assert plain[np.isinf(ALL_FP16)].all()


def test_rounding_up_is_needed():
    # rounding t to nearest instead of up would flag |x| = 6.0 at t = 6.001
    x = np.float16(6.0)
    assert not (np.float64(x) >= 6.001)
    assert np.float16(6.001) == x                     # nearest fp16 is 6.0 ...
    assert smallest_fp16_at_or_above(6.001) > 6.0     # ... the rule uses the next one up
