"""bench.py's clock record and peaks (no GPU). The sampler reads nvidia-smi's CSV samples,
reports the median SM clock under load, the largest maximum clock and every throttle reason
seen active, skips lines it cannot read, and says so when nvidia-smi is missing; a fake
nvidia-smi on PATH prints the samples and changes no setting of any GPU. The HBM peak comes
from the measured peaks file when there is one, else from the stated fallback."""

import os
import time

import bench


def _fake_smi(tmp_path, lines):
    exe = tmp_path / "nvidia-smi"
    body = "".join(f"printf '%s\\n' '{ln}'\n" for ln in lines)
    exe.write_text("#!/bin/sh\n" + body + "exec sleep 30\n")
    exe.chmod(0o755)
    return str(tmp_path)


def _sample(monkeypatch, tmp_path, lines):
    monkeypatch.setenv("PATH", _fake_smi(tmp_path, lines) + os.pathsep + os.environ["PATH"])
    s = bench.ClockSampler(0)
    s.start()
    deadline = time.time() + 10
    while len(s.lines) < len(lines) and time.time() < deadline:
        time.sleep(0.05)
    return s.stop()


def test_median_clock_and_the_power_cap_reason(monkeypatch, tmp_path):
    got = _sample(monkeypatch, tmp_path, [
        "1965, 1965, Not Active, Not Active, Not Active, Not Active",
        "1950, 1965, Not Active, Not Active, Not Active, Active",
        "1905, 1965, Not Active, Not Active, Not Active, Active",
    ])
    assert got["sm_mhz"] == 1950 and got["sm_max_mhz"] == 1965
    assert got["reasons"] == ["sw_power_cap"] and got["samples"] == 3


def test_every_slowdown_reason_is_reported_and_bad_lines_are_skipped(monkeypatch, tmp_path):
    got = _sample(monkeypatch, tmp_path, [
        "1200, 1965, Active, Not Active, Not Active, Not Active",
        "[N/A], [N/A], Not Active, Not Active, Not Active, Not Active",
        "1300, 1965, Not Active, Active, Active, Not Active",
        "garbled",
    ])
    assert got["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
    assert got["samples"] == 2 and got["sm_mhz"] == 1250


def test_missing_nvidia_smi_is_stated(monkeypatch, tmp_path):
    monkeypatch.setenv("PATH", str(tmp_path))  # an empty directory: no nvidia-smi
    s = bench.ClockSampler(0)
    s.start()
    got = s.stop()
    assert got["sm_mhz"] is None and got["reasons"] == ["nvidia-smi unavailable"]


def test_peaks_come_from_the_measured_file_else_the_stated_fallback(monkeypatch, tmp_path):
    # with no measured file the HBM denominator is the fallback 6.65 TB/s, labelled so
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.peaks() == {"hbm_gbs": 6650.0, "src": "fallback"}
    (tmp_path / "MEASURED_PEAKS.json").write_text('{"hbm_gbs": 6541.8}')
    assert bench.peaks() == {"hbm_gbs": 6541.8, "src": "measured"}
