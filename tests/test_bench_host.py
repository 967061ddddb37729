"""Host-side rules of bench.py (no GPU)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _clocks(sm, mx, reasons):
    return {"sm_mhz": sm, "sm_max_mhz": mx, "reasons": reasons, "samples": 5}


def test_clean_and_power_capped_runs_are_kept():
    assert not bench.clocks_rejected(_clocks(1965.0, 1965.0, []))
    assert not bench.clocks_rejected(_clocks(1852.0, 1965.0, ["sw_power_cap"]))
    # a dense step settling far down under the power cap is still a valid run
    assert not bench.clocks_rejected(_clocks(1300.0, 1965.0, ["sw_power_cap"]))
    assert not bench.clocks_rejected(None)


def test_slowdowns_and_leftover_clock_locks_are_measured_again():
    for reason in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"):
        assert bench.clocks_rejected(_clocks(1965.0, 1965.0, [reason]))
        assert bench.clocks_rejected(_clocks(1500.0, 1965.0, ["sw_power_cap", reason]))
    # well below the maximum with nothing to explain it: a lock someone left behind
    assert bench.clocks_rejected(_clocks(1100.0, 1965.0, []))
    assert not bench.clocks_rejected(_clocks(1800.0, 1965.0, []))
