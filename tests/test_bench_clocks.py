"""bench.py's clock sampler against a stand-in nvidia-smi that prints the
query's CSV rows (no GPU): samples inside the timed region are kept, the
median SM clock and the active throttle reasons are reported."""
import os
import stat
import sys
import time

import bench

FAKE = r'''#!{python}
import datetime, sys, time
for i in range(400):
    now = datetime.datetime.now().strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    sm = 1965 if i % 2 else 1950
    cap = "Active" if i % 5 == 0 else "Not Active"
    print(f"{{now}}, {{sm}}, 1965, 251.5, 0x0000000000000004, Not Active, Not Active, Not Active, {{cap}}", flush=True)
    time.sleep(0.02)
'''


def test_clock_sampler_parses_the_timed_window(tmp_path, monkeypatch):
    exe = tmp_path / "nvidia-smi"
    exe.write_text(FAKE.format(python=sys.executable))
    exe.chmod(exe.stat().st_mode | stat.S_IEXEC)
    monkeypatch.setenv("PATH", f"{tmp_path}{os.pathsep}{os.environ['PATH']}")
    s = bench.ClockSampler(None)
    s.start()
    time.sleep(0.2)
    s.mark_start()
    time.sleep(0.6)
    s.mark_end()
    out = s.stop()
    assert 10 <= out["samples"] <= 60
    assert out["sm_mhz"] in (1950.0, 1957.5, 1965.0)
    assert out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]
    assert out["power_w_max"] == 251.5


def test_clock_sampler_without_nvidia_smi(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", str(tmp_path))
    s = bench.ClockSampler(None)
    s.start()
    s.mark_start()
    s.mark_end()
    out = s.stop()
    assert out["reasons"] == ["unavailable"] and out["sm_mhz"] is None
    assert not os.path.exists(s.path)  # no sample file left behind
