"""bench.py's clock record on CPU, against a stand-in nvidia-smi that prints
the same CSV fields: only samples inside the timed window count, the median
SM clock comes from the busy samples, and a throttle reason is reported only
when its field reads "Active"."""
import os
import stat
import sys
import time

import bench

FAKE = r'''#!PYTHON
import datetime, sys, time
n = 0
while True:
    now = datetime.datetime.now().strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    sm = 1965 if n % 4 else 1900
    print(f"{now}, 0, {sm}, 1965, 900.5, 0x0000000000000004, Not Active, Not Active, "
          f"Not Active, Active", flush=True)
    n += 1
    time.sleep(0.05)
'''


def _fake_smi(tmp_path, monkeypatch):
    exe = tmp_path / "nvidia-smi"
    exe.write_text(FAKE.replace("PYTHON", sys.executable))
    exe.chmod(exe.stat().st_mode | stat.S_IEXEC)
    monkeypatch.setenv("PATH", str(tmp_path) + os.pathsep + os.environ["PATH"])


def test_clock_record_from_samples_inside_the_window(tmp_path, monkeypatch):
    _fake_smi(tmp_path, monkeypatch)
    c = bench.ClockSampler(0).start()
    time.sleep(0.2)             # samples before the window are dropped
    c.mark(True)
    time.sleep(0.5)
    c.mark(False)
    rec = c.stop()
    assert rec is not None
    assert rec["sm_max_mhz"] == 1965.0
    assert rec["sm_mhz"] == 1965.0            # median of 1965 x3 : 1900 x1
    assert rec["reasons"] == ["sw_power_cap"]  # "Not Active" fields are not reasons
    assert 3 <= rec["samples"] <= 16
    assert rec["in_window"] == rec["samples"]
    assert 450 <= rec["window_ms"] <= 3000


def test_window_shorter_than_the_interval_takes_the_nearest_samples(tmp_path, monkeypatch):
    """A timed region between two samples: the sample before it and the one
    after it stand in, and the record says none fell inside."""
    _fake_smi(tmp_path, monkeypatch)
    c = bench.ClockSampler(0).start()
    time.sleep(0.3)
    # the stand-in prints every 50 ms: a 1 ms window right after a sample
    # holds none
    c.mark(True)
    c.mark(False)
    c.t0 = c.t1 = time.time() - 0.1
    c.t1 += 0.001
    time.sleep(0.2)
    rec = c.stop()
    assert rec is not None
    assert rec["sm_max_mhz"] == 1965.0
    assert 1 <= rec["samples"] <= 2
    assert rec["in_window"] <= 1


def test_no_nvidia_smi_gives_no_record(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", str(tmp_path))
    c = bench.ClockSampler(0).start()
    c.mark(True)
    c.mark(False)
    assert c.stop() is None
