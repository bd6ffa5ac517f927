"""Host logic of bench.py that needs no GPU: the clock summary.

nvidia-smi samples carry timestamps; the summary takes those inside the timed
region, or, when the region held none (it is shorter than the sampling
period), those of the window of the same steps run right after it."""
import datetime
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _row(t, mhz, power_cap=False, hw=False):
    stamp = datetime.datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    na, a = "Not Active", "Active"
    return [stamp, "0", str(mhz), "1965", "900.0", "0x0", a if hw else na, na, na, a if power_cap else na]


def test_clock_summary_prefers_samples_inside_the_timed_region():
    t = 1.0e9
    rows = [_row(t + 0.05, 1965), _row(t + 0.30, 1800, power_cap=True), _row(t + 0.60, 1700, power_cap=True)]
    c = bench.summarize_clocks(rows, t + 0.25, t + 0.35, t + 0.75)
    assert c["window"] == "timed region"
    assert c["samples_in_timed_region"] == 1 and c["samples"] == 1
    assert c["sm_mhz"] == 1800 and c["sm_max_mhz"] == 1965
    assert c["reasons"] == ["sw_power_cap"]


def test_clock_summary_falls_back_to_the_window_after_a_short_region():
    t = 1.0e9
    rows = [_row(t + 0.05, 1965), _row(t + 0.50, 1710, power_cap=True), _row(t + 0.70, 1690, hw=True)]
    c = bench.summarize_clocks(rows, t + 0.10, t + 0.14, t + 0.80)
    assert c["samples_in_timed_region"] == 0 and c["samples"] == 2
    assert c["window"].startswith("the same steps")
    assert c["sm_mhz"] == 1700
    # a slowdown seen in the window is reported (such a run is re-measured)
    assert c["reasons"] == ["hw_slowdown", "sw_power_cap"]


def test_clock_summary_without_times_uses_every_sample():
    rows = [_row(1.0e9, 1965), _row(1.0e9 + 0.1, 1900)]
    c = bench.summarize_clocks(rows)
    assert c["window"] == "sampler run" and c["samples"] == 2 and c["sm_mhz"] == 1932.5
    assert bench.summarize_clocks([]) is None
