"""bench.py's clock record on CPU: the sampler's child protocol with a fake
child (no NVML here), and its fallback when no sampler can start."""
import os
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402

# stands in for the NVML child: the same protocol ("ready <max MHz>", then one
# "<monotonic time> <MHz> <reason bits>" row per sample once stdin closes),
# with one row before and one after the parent's bracket
_FAKE_CHILD = r"""
import select, sys, time
print("ready 1965", flush=True)
rows = ["%.6f %d %d" % (time.monotonic() - 100.0, 1000, 0x8)]
while not select.select([sys.stdin], [], [], 0)[0]:
    rows.append("%.6f %d %d" % (time.monotonic(), 1965, 0x4 | 0x1))
    time.sleep(0.001)
rows.append("%.6f %d %d" % (time.monotonic() + 100.0, 900, 0x40))
sys.stdout.write("\n".join(rows) + "\n")
"""


def test_sampler_keeps_the_samples_inside_the_bracket(monkeypatch):
    monkeypatch.setattr(bench, "_SAMPLER_CHILD", _FAKE_CHILD)
    cs = bench.ClockSampler(0)
    with cs:
        time.sleep(0.05)
    s = cs.summary()
    # the rows at t - 100 s (hw_slowdown, 1000 MHz) and t + 100 s
    # (hw_thermal_slowdown, 900 MHz) fall outside; gpu_idle is not a reason
    assert s["sm_max_mhz"] == 1965 and s["sm_mhz"] == 1965, s
    assert s["samples"] >= 5 and s["reasons"] == ["sw_power_cap"], s


def test_sampler_without_nvml_reports_no_clocks(monkeypatch):
    monkeypatch.setattr(bench, "_SAMPLER_CHILD", "import sys; sys.exit(3)")
    cs = bench.ClockSampler(0)
    with cs:
        pass
    assert cs.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
