"""bench.py's clock sampler against a stand-in nvidia-smi on PATH (CPU only):
the sample taken before the timed region is dropped, the rest are parsed
into the median SM clock, the max clock and the active throttle reasons."""
import os
import stat
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

FAKE = """#!/bin/sh
echo "0, 100, 1965, 500.0, 0x0, Not Active, Not Active, Not Active, Not Active"
while true; do
  echo "0, 1900, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, Active"
  sleep 0.02
done
"""


def test_sampler_drops_the_first_sample_and_parses_reasons(tmp_path, monkeypatch):
    exe = tmp_path / "nvidia-smi"
    exe.write_text(FAKE)
    exe.chmod(exe.stat().st_mode | stat.S_IEXEC)
    monkeypatch.setenv("PATH", str(tmp_path) + os.pathsep + os.environ["PATH"])
    import bench
    s = bench.ClockSampler(0)
    s.start()
    time.sleep(0.2)
    c = s.stop()
    assert c["samples"] >= 2
    assert c["sm_mhz"] == 1900.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"]


def test_sampler_without_nvidia_smi(monkeypatch, tmp_path):
    monkeypatch.setenv("PATH", str(tmp_path))
    import bench
    s = bench.ClockSampler(0)
    s.start()
    assert s.stop()["sm_mhz"] is None
