"""bench.py's clock sampler on the host, driven by a stand-in for nvidia-smi
that prints the same CSV fields (no GPU): the summary covers the samples
inside the marked timed region, throttle reasons come from every sample,
and a missing tool reads as unsampled."""

import os
import sys
import time

import bench

# Prints one CSV row per period like `nvidia-smi --query-gpu=... -lms P`:
# 1000 MHz with sw_power_cap active until the flag file exists, then 1965 MHz
# with no reason active.
FAKE = '''#!{python}
import datetime, os, sys, time
period = int(sys.argv[sys.argv.index("-lms") + 1]) / 1000.0
flag = {flag!r}
while True:
    hot = os.path.exists(flag)
    sm = 1965 if hot else 1000
    cap = "Not Active" if hot else "Active"
    ts = datetime.datetime.now().strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    print(f"0, {{sm}}, 1965, 700.00, 0x0, Not Active, Not Active, Not Active, {{cap}}, {{ts}}",
          flush=True)
    time.sleep(period)
'''


def make_fake(tmp_path):
    flag = tmp_path / "hot"
    tool = tmp_path / "fake-smi"
    tool.write_text(FAKE.format(python=sys.executable, flag=str(flag)))
    tool.chmod(0o755)
    return str(tool), flag


def test_summary_covers_the_timed_region(tmp_path, monkeypatch):
    monkeypatch.setenv("MALA_BENCH_OUT", str(tmp_path))
    tool, flag = make_fake(tmp_path)
    c = bench.ClockSampler(0, tool=tool)
    c.start()
    assert os.path.getsize(c.path) > 0  # start() waited for the first sample
    time.sleep(0.3)                      # "warm-up" at the low clock
    flag.write_text("1")
    time.sleep(0.12)
    c.mark("begin")
    time.sleep(0.5)                      # "timed region" at the full clock
    c.mark("end")
    out = c.stop()
    assert out["window"] == "timed region"
    assert out["samples"] >= 4
    assert out["sm_mhz"] == 1965.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]  # seen during the warm-up


def test_without_marks_every_sample_counts(tmp_path, monkeypatch):
    monkeypatch.setenv("MALA_BENCH_OUT", str(tmp_path))
    tool, _ = make_fake(tmp_path)
    c = bench.ClockSampler(0, tool=tool)
    c.start()
    time.sleep(0.2)
    out = c.stop()
    assert out["window"].startswith("whole run")
    assert out["samples"] >= 2 and out["sm_mhz"] == 1000.0


def test_missing_tool_reads_as_unsampled(tmp_path, monkeypatch):
    monkeypatch.setenv("MALA_BENCH_OUT", str(tmp_path))
    c = bench.ClockSampler(0, tool=str(tmp_path / "no-such-tool"))
    c.start()
    assert c.stop() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
