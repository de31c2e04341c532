"""bench.py's clock sampler on the CPU, against a fake nvidia-smi that prints
one CSV sample every 25 ms: only samples stamped inside the timed region count,
throttle reasons are picked up, and a missing nvidia-smi reads as unavailable."""
import os
import stat
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

FAKE = """#!{py}
import datetime, os, time
cap = os.environ.get("FAKE_POWER_CAP", "Not Active")
while True:
    ts = datetime.datetime.now().strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    print(ts + ", 1965, 1965, 512.30, 0x0000000000000000, Not Active, Not Active, Not Active, " + cap, flush=True)
    time.sleep(0.025)
"""


def _fake_smi(tmp_path, monkeypatch):
    exe = tmp_path / "nvidia-smi"
    exe.write_text(FAKE.format(py=sys.executable))
    exe.chmod(exe.stat().st_mode | stat.S_IEXEC)
    monkeypatch.setenv("PATH", str(tmp_path) + os.pathsep + os.environ["PATH"])


def _run(sampler, warm=0.4, timed=0.3, after=0.2):
    sampler.start()
    time.sleep(warm)
    sampler.begin()
    time.sleep(timed)
    sampler.end()
    time.sleep(after)
    sampler.stop()
    return sampler.summary()


def test_samples_inside_the_timed_region_only(tmp_path, monkeypatch):
    _fake_smi(tmp_path, monkeypatch)
    s = bench.ClockSampler(0)
    out = _run(s)
    assert out["sm_mhz"] == 1965.0 and out["sm_max_mhz"] == 1965.0 and out["reasons"] == []
    # 0.3 s of 25 ms samples (+ one interval of slack each side), not the 0.9 s the process ran
    assert 6 <= out["samples"] <= 16, out
    assert len(s.lines) > out["samples"] + 8


def test_power_cap_reason_is_reported(tmp_path, monkeypatch):
    _fake_smi(tmp_path, monkeypatch)
    monkeypatch.setenv("FAKE_POWER_CAP", "Active")
    out = _run(bench.ClockSampler(0), warm=0.3, timed=0.2, after=0.1)
    assert out["reasons"] == ["sw_power_cap"] and out["samples"] > 0


def test_missing_nvidia_smi_reads_as_unavailable(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", str(tmp_path))
    out = _run(bench.ClockSampler(0), warm=0.0, timed=0.05, after=0.0)
    assert out == {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}


def test_sampler_queries_the_visible_gpu(monkeypatch):
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "5,GPU-1234")
    assert bench.ClockSampler(0).index == "5" and bench.ClockSampler(1).index == "GPU-1234"
    monkeypatch.delenv("CUDA_VISIBLE_DEVICES")
    assert bench.ClockSampler(0).index == "0"
