"""Host-side pieces of bench.py that need no GPU: the load window and the clock-record parser."""
import os
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_keep_busy_runs_for_the_window_and_ends_synchronised():
    calls = []

    def step():
        calls.append("step")
        time.sleep(0.002)

    def sync():
        calls.append("sync")

    t0 = time.perf_counter()
    n = bench.keep_busy(step, 0.05, sync)
    dt = time.perf_counter() - t0
    assert n == calls.count("step") and n >= 8
    assert dt >= 0.05
    assert calls[-1] == "sync"


def test_keep_busy_with_no_window_still_runs_one_batch():
    n = bench.keep_busy(lambda: None, 0.0, lambda: None)
    assert n == 8


class _DoneProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def _record(lines):
    s = bench.ClockSampler(0)
    s.proc = _DoneProc()
    s.lines = lines
    return s.stop()


def test_clock_record_median_max_and_reasons():
    lines = [
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1350, 1965, 998.7, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1950, 1965, 990.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
        "0, [N/A], 1965, 990.0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    rec = _record(lines)
    assert rec["samples"] == 3
    assert rec["sm_mhz"] == 1950.0 and rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["sw_power_cap"]


def test_clock_record_flags_thermal_slowdown():
    rec = _record(["0, 1200, 1965, 1000, 0x40, Not Active, Active, Not Active, Not Active"])
    assert rec["reasons"] == ["hw_thermal_slowdown"]


def test_clock_record_without_nvidia_smi():
    s = bench.ClockSampler(0)
    assert s.stop()["reasons"] == ["nvidia-smi unavailable"]
