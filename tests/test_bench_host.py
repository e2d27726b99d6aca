"""Host-side pieces of bench.py that need no GPU: the clock sampler's time-window summary."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))


def test_clock_summary_keeps_only_the_window():
    import bench
    cs = bench.ClockSampler(0)
    cs.proc = object()   # pretend nvidia-smi started; rows are injected below
    cs.rows = [(0.5, 1965.0, 1965.0, set()),                   # idle, before the window
               (1.1, 1740.0, 1965.0, {"sw_power_cap"}),
               (1.2, 1750.0, 1965.0, {"sw_power_cap"}),
               (1.3, 1760.0, 1965.0, set()),
               (2.5, 1965.0, 1965.0, set())]                   # idle, after the window
    got = cs.summary(1.0, 2.0)
    assert got["samples"] == 3
    assert got["sm_mhz"] == 1750.0
    assert got["sm_max_mhz"] == 1965.0
    assert got["reasons"] == ["sw_power_cap"]
    empty = cs.summary(3.0, 4.0)
    assert empty["samples"] == 0 and empty["sm_mhz"] is None


def test_clock_summary_without_nvidia_smi():
    import bench
    cs = bench.ClockSampler(0)
    got = cs.summary(0.0, 1.0)
    assert got["reasons"] == ["nvidia-smi unavailable"] and got["samples"] == 0
