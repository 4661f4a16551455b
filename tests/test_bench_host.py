"""Host-side arithmetic of bench.py (no GPU): the refresh share and the roofline entries."""

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_refresh_share_from_per_step_times():
    # steps t = 3 .. 18 with refresh every 8: t = 8 and t = 16 refresh
    step_ms = [1.0] * 16
    step_ms[8 - 3] = 1.8
    step_ms[16 - 3] = 2.2
    r, n, share = bench.refresh_share(step_ms, 3, 8)
    assert r == pytest.approx(2.0) and n == pytest.approx(1.0)
    assert share == pytest.approx((2.0 - 1.0) / (8 * 1.0))
    # every step refreshes: no reuse step to compare with
    r, n, share = bench.refresh_share([2.0, 2.0], 0, 1)
    assert r == 2.0 and n is None and share is None


def test_kernel_roofline_units_and_fraction():
    # three launches, 3 ms in all, 3 * 1e12 flops: 1000 TFLOP/s against a 2000 peak
    e = bench.kernel_roofline(3.0, 3, 3e12, 2000.0, "TFLOP/s", "tensor", "k", "basis")
    assert e["achieved"] == 1000.0 and e["frac"] == 0.5 and e["us_per_launch"] == 1000.0
    # bytes: 367 MB in 60 us -> 6116.7 GB/s
    e = bench.kernel_roofline(0.06, 1, 367e6, 6546.9, "GB/s", "hbm", "k", "basis")
    assert e["achieved"] == pytest.approx(6116.7, abs=0.1) and e["frac"] == pytest.approx(0.9343, abs=1e-4)
    e = bench.kernel_roofline(0.0, 0, 0.0, 6546.9, "GB/s", "hbm", "k", "basis")
    assert e["achieved"] is None and e["frac"] is None
