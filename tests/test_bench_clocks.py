"""The clock sampler of the benchmark (bench.Clocks), run on the CPU against a
stand-in for nvidia-smi that prints one CSV sample every 20 ms with the time
since its start as the SM clock: only the samples written after the timed
region's start count, the median and the maximum clock come from them, and
a throttle reason is reported only if it was active in one of them."""
import os
import stat
import time

import bench

# sample 0 (before the timed region) reports hw_slowdown; samples from 300 ms
# on report sw_power_cap
FAKE = r"""#!/usr/bin/env python3
import time
t0 = time.time()
i = 0
while True:
    ms = int((time.time() - t0) * 1000)
    hw = "Active" if i == 0 else "Not Active"
    cap = "Active" if ms >= 300 else "Not Active"
    print(f"0, {ms}, 1965, 700.0, 0x0, {hw}, Not Active, Not Active, {cap}", flush=True)
    i += 1
    time.sleep(0.02)
"""


def test_samples_after_mark_only(tmp_path, monkeypatch):
    exe = tmp_path / "nvidia-smi"
    exe.write_text(FAKE)
    exe.chmod(exe.stat().st_mode | stat.S_IEXEC)
    monkeypatch.setenv("PATH", f"{tmp_path}{os.pathsep}{os.environ['PATH']}")
    ck = bench.Clocks(0)
    assert ck.p is not None and os.path.getsize(ck.f.name) > 0  # running before the warm-up
    time.sleep(0.2)
    ck.mark()
    time.sleep(0.4)
    r = ck.stop()
    assert r["samples"] >= 5
    assert r["sm_mhz"] >= 200  # no sample of the first 0.2 s counted
    assert r["sm_max_mhz"] == 1965
    assert r["reasons"] == ["sw_power_cap"]  # the hw_slowdown sample came before mark()


def test_missing_tool_reports_unavailable(monkeypatch, tmp_path):
    monkeypatch.setenv("PATH", str(tmp_path))
    ck = bench.Clocks(0)
    ck.mark()
    r = ck.stop()
    assert r["sm_mhz"] is None and r["reasons"] == ["nvidia-smi unavailable"]
