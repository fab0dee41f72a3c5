"""The bench's clock record (bench.ClockSampler) on synthetic samples: which
throttle reasons it reports, which samples count (those inside the timed
region) and how nvidia-smi's CSV lines are read.  A run is rejected or kept on
these fields, so they are checked without a GPU."""
from __future__ import annotations

import io
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _sampler(samples):
    s = bench.ClockSampler(0)
    s.samples = list(samples)
    return s


def test_summary_of_samples_inside_the_timed_region():
    R = bench.ClockSampler.REASONS
    s = _sampler([(1200.0, 1965.0, R["hw_slowdown"], 0.5),      # before the region: dropped
                  (1965.0, 1965.0, 0, 1.0),
                  (1905.0, 1965.0, R["sw_power_cap"], 1.5),
                  (1965.0, 1965.0, 0, 2.0),
                  (900.0, 1965.0, R["sw_thermal_slowdown"], 3.5)])  # after it: dropped
    rec = s.stop(1.0, 2.0)
    assert rec["samples"] == 3 and rec["sm_mhz"] == 1965.0 and rec["sm_min_mhz"] == 1905.0
    assert rec["sm_max_mhz"] == 1965.0 and rec["reasons"] == ["sw_power_cap"]


def test_every_reason_is_reported_and_empty_windows_keep_all_samples():
    R = bench.ClockSampler.REASONS
    s = _sampler([(1500.0, 1965.0, R["hw_slowdown"] | R["hw_thermal_slowdown"], 1.0),
                  (1600.0, 1965.0, R["sw_thermal_slowdown"], 2.0)])
    rec = s.stop(5.0, 6.0)            # no sample inside: the summary uses all of them
    assert rec["samples"] == 2 and rec["sm_mhz"] == 1550.0
    assert rec["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
    assert bench.ClockSampler(0).stop() is None


def test_nvidia_smi_lines():
    s = bench.ClockSampler(0)

    class _Fake:
        stdout = io.StringIO(
            "0, 1965, 1965, 650.2, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n"
            "0, 1800, 1965, 998.7, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n"
            "0, 1200, 1965, 700.0, 0x0000000000000048, Active, Active, Not Active, Not Active\n"
            "garbage line\n"
            "0, [N/A], 1965, 1.0, 0x0, Not Active, Not Active, Not Active, Not Active\n")
    s._smi = _Fake()
    s._read_smi()
    R = bench.ClockSampler.REASONS
    assert [(x[0], x[1], x[2]) for x in s.samples] == [
        (1965.0, 1965.0, 0), (1800.0, 1965.0, R["sw_power_cap"]),
        (1200.0, 1965.0, R["hw_slowdown"] | R["hw_thermal_slowdown"])]


def test_peaks_measured_file_or_labelled_fallback(tmp_path, monkeypatch):
    """The roofline's denominators: the driver's measured file when present
    (labelled "measured"), else the pool's earlier measurement (6.65 TB/s copy,
    1.59 PFLOP/s bf16 burst), labelled "fallback"."""
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    d, src = bench.measured_peaks()
    assert src == "fallback" and d["hbm_gbs"] == 6650.0 and d["bf16_tflops"] == 1590.0
    (tmp_path / "MEASURED_PEAKS.json").write_text('{"hbm_gbs": 6542.7, "bf16_tflops": 1628.3}')
    d, src = bench.measured_peaks()
    assert src == "measured" and d == {"hbm_gbs": 6542.7, "bf16_tflops": 1628.3}
