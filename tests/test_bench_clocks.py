"""The bench's clock sampler on the host, against a stand-in `nvidia-smi`.

The timed region of a short bench run lasts tens of milliseconds, so the
sampler must be polling before the region starts and must count only the
samples taken inside it.  A small script on PATH plays nvidia-smi's CSV loop
(one line per period, like the real `--query-gpu ... -lms` output); the tests
check that entering the sampler waits for the first line, that lines written
before entry are not counted as the region's, and that the throttle reasons
and clocks are read from the right columns.  No GPU is involved.
"""
import os
import stat
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _fake_smi(tmp_path, lines, period_s, start_delay_s=0.0):
    """An executable named nvidia-smi that prints `lines` (cycling the last one)
    every `period_s` after `start_delay_s`, until killed."""
    path = tmp_path / "nvidia-smi"
    body = "\n".join([
        "#!" + sys.executable,
        "import sys, time",
        f"time.sleep({start_delay_s})",
        f"lines = {lines!r}",
        "i = 0",
        "while True:",
        "    print(lines[min(i, len(lines) - 1)], flush=True)",
        "    i += 1",
        f"    time.sleep({period_s})",
    ])
    path.write_text(body + "\n")
    path.chmod(path.stat().st_mode | stat.S_IEXEC)
    return path


def _row(sm, smax=1965, power=900, cap="Not Active", thermal="Not Active"):
    return f"0, {sm}, {smax}, {power}, 0x0, Not Active, Not Active, {thermal}, {cap}"


def test_sampler_waits_for_the_first_sample_and_counts_the_region_only(tmp_path, monkeypatch):
    # a slow-starting poller: the first line comes 0.3 s after launch
    _fake_smi(tmp_path, [_row(345), _row(1965)], period_s=0.01, start_delay_s=0.3)
    monkeypatch.setenv("PATH", str(tmp_path) + os.pathsep + os.environ["PATH"])
    t0 = time.time()
    with bench.ClockSampler(0) as c:
        entered = time.time() - t0
        time.sleep(0.1)   # the timed region
    s = c.summary()
    assert entered >= 0.25            # it waited for the poller's first line
    assert s["samples"] >= 3          # lines written during the region
    assert s["sm_mhz"] == 1965.0      # the pre-region (idle) line is not counted
    assert s["sm_max_mhz"] == 1965.0 and s["reasons"] == []
    assert "note" not in s


def test_sampler_reports_throttle_reasons(tmp_path, monkeypatch):
    _fake_smi(tmp_path, [_row(1860, cap="Active"), _row(1860, cap="Active", thermal="Active")], period_s=0.01)
    monkeypatch.setenv("PATH", str(tmp_path) + os.pathsep + os.environ["PATH"])
    with bench.ClockSampler(0) as c:
        time.sleep(0.08)
    s = c.summary()
    assert s["sm_mhz"] == 1860.0
    assert s["reasons"] == ["sw_power_cap", "sw_thermal_slowdown"]


def test_sampler_without_nvidia_smi_says_unsampled(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", str(tmp_path))   # no nvidia-smi anywhere (nor stdbuf)
    with bench.ClockSampler(0) as c:
        pass
    assert c.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
