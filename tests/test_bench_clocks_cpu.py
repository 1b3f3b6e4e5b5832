"""bench.py's clock record on CPU: ClockSampler runs `nvidia-smi --query-gpu`
in the background during the timed region and reduces its CSV to the median
SM clock under load, the maximum clock and the throttle reasons seen.  A fake
`nvidia-smi` on PATH stands in for the real one (no GPU, no NVML)."""
import os
import stat
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

# index, clocks.sm, clocks.max.sm, power.draw, active mask, hw_slowdown,
# hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap
_LINES = [
    "0, 1590, 1965, 980.1, 0x4, Not Active, Not Active, Not Active, Active",
    "0, 1650, 1965, 990.5, 0x4, Not Active, Not Active, Not Active, Active",
    "0, 1700, 1965, 1000.0, 0x0, Not Active, Not Active, Not Active, Not Active",
    "0, 345, 1965, 120.0, 0x1, Not Active, Not Active, Not Active, Not Active",
    "garbage line",
]


def _fake_smi(tmp_path, lines):
    exe = tmp_path / "nvidia-smi"
    body = "\n".join(f"echo '{ln}'" for ln in lines)
    exe.write_text(f"#!/bin/sh\n{body}\nsleep 30\n")
    exe.chmod(exe.stat().st_mode | stat.S_IEXEC)
    return str(tmp_path)


def _sample(tmp_path, monkeypatch, lines):
    monkeypatch.setenv("PATH", _fake_smi(tmp_path, lines) + os.pathsep + os.environ["PATH"])
    c = bench.ClockSampler(0)
    c.start()
    t0 = time.time()
    while time.time() - t0 < 5 and (not os.path.exists(c.path) or
                                    open(c.path).read().count("\n") < len(lines)):
        time.sleep(0.05)
    return c.stop()


def test_median_under_load_max_and_reasons(tmp_path, monkeypatch):
    r = _sample(tmp_path, monkeypatch, _LINES)
    assert r["samples"] == 4                       # the malformed line is skipped
    assert r["sm_mhz"] == 1650.0                   # idle 345 MHz sample left out
    assert r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"]


def test_slowdown_reasons_are_reported(tmp_path, monkeypatch):
    lines = ["0, 1200, 1965, 700.0, 0x8, Active, Not Active, Active, Not Active"]
    r = _sample(tmp_path, monkeypatch, lines)
    assert r["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert r["sm_mhz"] == 1200.0


def test_missing_nvidia_smi(monkeypatch, tmp_path):
    monkeypatch.setenv("PATH", str(tmp_path))      # an empty directory: no nvidia-smi
    c = bench.ClockSampler(0)
    c.start()
    r = c.stop()
    assert r["sm_mhz"] is None and r["reasons"] == ["nvidia-smi unavailable"]
