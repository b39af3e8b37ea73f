"""bench.ClockSampler against a fake nvidia-smi (CPU only): it waits for the
first sample, reports only what was sampled from mark() on, takes the
median clock, and lists the throttle reasons that were active."""
import os
import stat
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

FAKE = """#!/bin/sh
# prints one sample line at a time, like 'nvidia-smi --query-gpu=... -lms N'
i=0
while [ $i -lt 400 ]; do
  if [ $i -lt 2 ]; then echo "1200, 1965, 300.0, Not Active, Not Active, Not Active, Not Active";
  elif [ $i -eq 3 ]; then echo "1965, 1965, 950.0, Not Active, Not Active, Not Active, Active";
  else echo "1965, 1965, 900.0, Not Active, Not Active, Not Active, Not Active"; fi
  i=$((i+1)); sleep 0.02
done
"""


@pytest.fixture
def fake_smi(tmp_path, monkeypatch):
    p = tmp_path / "nvidia-smi"
    p.write_text(FAKE)
    p.chmod(p.stat().st_mode | stat.S_IEXEC)
    monkeypatch.setenv("PATH", str(tmp_path) + os.pathsep + os.environ["PATH"])
    monkeypatch.setattr(bench.torch.cuda, "get_device_properties",
                        lambda dev: type("P", (), {"uuid": "GPU-00000000-fake"})())
    monkeypatch.setattr(bench.torch.cuda, "synchronize", lambda *a, **k: None)
    return p


def test_samples_from_mark_on(fake_smi):
    c = bench.ClockSampler(0)
    c.start()
    assert c.count() >= 1          # running before anything is timed
    import time
    time.sleep(0.08)               # the pre-region samples (1200 MHz) are skipped
    c.mark()
    calls = []
    c.keep_loaded(lambda: calls.append(1) or time.sleep(0.01), min_samples=5, max_s=2.0)
    r = c.stop()
    assert r["samples"] >= 5 and r["sm_mhz"] == 1965.0 and r["sm_max_mhz"] == 1965.0
    assert calls and "untimed" in r["window"]


def test_reasons_and_unsampled(fake_smi):
    c = bench.ClockSampler(0)
    c.start()
    c.mark()
    c.base = 0                     # include every sample, the power-cap one among them
    import time
    time.sleep(0.2)
    r = c.stop()
    assert r["reasons"] == ["sw_power_cap"] and r["window"] == "the timed region"
    none = bench.ClockSampler(0)   # never started: reported as unsampled
    assert none.stop()["reasons"] == ["unsampled"]
