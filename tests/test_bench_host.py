"""Host-side pieces of the bench on CPU: the clock sampler's parsing of nvidia-smi's
CSV (against a fake nvidia-smi on PATH) and the peak table's fallback."""
import json
import os
import stat
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

FAKE = """#!/bin/sh
# prints what `nvidia-smi --query-gpu=... --format=csv,noheader,nounits -lms 200` would
echo "0, 1965, 1965, 640.5, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active"
echo "0, 1800, 1965, 990.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active"
echo "0, 1965, 1965, 700.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active"
echo "garbage line"
exec sleep 30
"""


def test_clock_sampler_parses_samples_and_reasons(tmp_path, monkeypatch):
    exe = tmp_path / "nvidia-smi"
    exe.write_text(FAKE)
    exe.chmod(exe.stat().st_mode | stat.S_IEXEC)
    monkeypatch.setenv("PATH", f"{tmp_path}{os.pathsep}{os.environ['PATH']}")
    cs = bench.ClockSampler(0)
    cs.start()
    time.sleep(0.5)
    out = cs.stop()
    assert out["samples"] == 3
    assert out["sm_mhz"] == 1965.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]


def test_clock_sampler_without_nvidia_smi(monkeypatch, tmp_path):
    monkeypatch.setenv("PATH", str(tmp_path))          # nothing to run
    cs = bench.ClockSampler(0)
    cs.start()
    out = cs.stop()
    assert out["sm_mhz"] is None and out["reasons"] == ["nvidia-smi unavailable"]


def test_peaks_measured_or_fallback(tmp_path, monkeypatch):
    peaks, src = bench.load_peaks()
    if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")):
        assert src == "measured" and float(peaks["hbm_gbs"]) > 0
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    peaks, src = bench.load_peaks()
    assert src == "fallback" and peaks == bench.PEAKS_FALLBACK
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 1.0, "bf16_tflops": 2.0}))
    peaks, src = bench.load_peaks()
    assert src == "measured" and peaks["hbm_gbs"] == 1.0
