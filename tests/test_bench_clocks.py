"""bench.py's clock sampler, run against a stand-in nvidia-smi on the CPU."""
import os
import stat
import sys
import time

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402

# index, clocks.sm, clocks.max.sm, power, active reasons, hw, hw_thermal, sw_thermal, sw_power_cap
_SCRIPT = """#!/bin/sh
sleep 0.3
while true; do
  echo "0, 1965, 1965, 612.5, 0x0000000000000000, Not Active, Not Active, Not Active, Active"
  sleep 0.01
done
"""


def _fake_smi(tmp_path, monkeypatch):
    exe = tmp_path / "nvidia-smi"
    exe.write_text(_SCRIPT)
    exe.chmod(exe.stat().st_mode | stat.S_IEXEC)
    monkeypatch.setenv("PATH", f"{tmp_path}{os.pathsep}{os.environ.get('PATH', '')}")


def test_sampler_waits_for_first_sample_and_parses(tmp_path, monkeypatch):
    _fake_smi(tmp_path, monkeypatch)
    s = bench.ClockSampler(0)
    t0 = time.monotonic()
    s.start()
    # start() returns only once the (slow-starting) sampler has printed a line
    assert time.monotonic() - t0 >= 0.25
    time.sleep(0.1)  # a short "timed region"
    c = s.stop()
    assert c["samples"] >= 3
    assert c["sm_mhz"] == 1965.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"]


def test_sampler_without_nvidia_smi(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", str(tmp_path))  # an empty directory: no nvidia-smi
    s = bench.ClockSampler(0)
    s.start()
    assert s.stop()["sm_mhz"] is None
