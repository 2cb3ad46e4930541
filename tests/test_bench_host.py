"""Host-side pieces of bench.py that need no GPU."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_clock_lines_summary():
    lines = [
        "1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "1950, 1965, 990.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "1300, 1965, 999.0, 0x0000000000000008, Active, Not Active, Not Active, Active",
        "garbled line",
        "[N/A], 1965, 1.0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    s = bench.parse_clock_lines(lines)
    assert s["samples"] == 3
    assert s["sm_mhz"] == 1950.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["hw_slowdown", "sw_power_cap"]


def test_clock_lines_empty():
    s = bench.parse_clock_lines([])
    assert s["sm_mhz"] is None and s["reasons"] == [] and s["samples"] == 0
