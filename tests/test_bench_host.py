"""The bench's host-side arithmetic on CPU: which GEMM peak a timed region is divided by, where
the peaks come from, when a committed DRAM-traffic capture still applies, how many rotating
buffer sets a back-to-back figure needs, the FP32 FMA roofline, and the flat map of secondary
roofline fractions."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

PK = {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
CAPPED = {"sm_mhz": 1760.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
FULL = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
LOCKED_LOW = {"sm_mhz": 1200.0, "sm_max_mhz": 1965.0, "reasons": []}


def test_short_region_takes_the_burst_peak_even_when_capped():
    # a region of milliseconds runs at burst clocks whatever one sample says
    assert bench.tensor_peak_for(PK, 0.0013, CAPPED) == (1600.0, "bf16_tflops")


def test_long_capped_region_takes_the_sustained_peak():
    assert bench.tensor_peak_for(PK, 3.0, CAPPED) == (1400.0, "bf16_tflops_sustained")
    # a median clock under 90 % of max counts as capped even with no reason reported
    assert bench.tensor_peak_for(PK, 3.0, LOCKED_LOW) == (1400.0, "bf16_tflops_sustained")


def test_long_region_at_full_clock_keeps_the_burst_peak():
    assert bench.tensor_peak_for(PK, 3.0, FULL) == (1600.0, "bf16_tflops")
    assert bench.tensor_peak_for(PK, 3.0, None) == (1600.0, "bf16_tflops")
    no_sustained = {k: v for k, v in PK.items() if k != "bf16_tflops_sustained"}
    assert bench.tensor_peak_for(no_sustained, 3.0, CAPPED) == (1600.0, "bf16_tflops")


def test_peaks_read_the_measured_file_else_the_fallback(tmp_path, monkeypatch):
    f = tmp_path / "peaks.json"
    f.write_text(json.dumps(PK))
    monkeypatch.setattr(bench, "PEAKS_FILE", str(f))
    d, which = bench.peaks()
    assert which == "of measured" and d["bf16_tflops"] == 1600.0
    monkeypatch.setattr(bench, "PEAKS_FILE", str(tmp_path / "absent.json"))
    d, which = bench.peaks()
    assert which == "of fallback" and d == bench.FALLBACK
    f.write_text("{not json")
    monkeypatch.setattr(bench, "PEAKS_FILE", str(f))
    assert bench.peaks()[1] == "of fallback"


def test_traffic_capture_applies_only_to_the_unchanged_source(tmp_path, monkeypatch):
    src = "igemm_rowt.cu"
    sha = bench.kernel_source_hash(src)
    assert len(sha) == 16
    rec = {"igemm_tc": {"source_sha": sha, "dram_bytes_per_launch": 123}}
    f = tmp_path / "traffic.json"
    f.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.traffic_for("igemm_tc", src)["dram_bytes_per_launch"] == 123
    assert bench.traffic_for("igemm_halo", src) is None          # no capture of that kernel
    rec["igemm_tc"]["source_sha"] = "0" * 16                     # kernel edited since
    f.write_text(json.dumps(rec))
    assert bench.traffic_for("igemm_tc", src) is None
    assert bench.kernel_source_hash("no_such_file.cu") == ""


@pytest.mark.parametrize("set_bytes", [1, 1 << 20, 64 << 20, 126 << 20, 300 << 20, 4 << 30])
def test_rotating_sets_exceed_twice_l2(set_bytes):
    n = bench.sets_for(set_bytes)
    assert n >= 2
    assert n * set_bytes > 2 * bench.L2_BYTES


def test_ffma_peak_is_lanes_times_clock():
    # 148 SMs x 128 FP32 lanes x 2 FLOP per FMA at 1965 MHz
    assert bench.ffma_peak_tflops(148, 1965.0) == pytest.approx(74.45, abs=0.01)
    assert bench.ffma_peak_tflops(1, 1000.0) == pytest.approx(0.256)


def test_compact_rooflines_names_and_skips():
    dwm = {"depthwise56_s1": {"frac": 0.7, "frac_b2b": 0.65},
           "dw1d_same_fwd": {"frac": 0.2},
           "dw1d_same_fwd_cudacore": {"frac": 0.19}}            # reported elsewhere
    more = {"ensemble": {"bound": "hbm", "frac": 0.38, "frac_b2b": 0.39},
            "sweep_direct": {"bound": "hbm", "frac": 0.01, "us": 19000.0},   # slow forced path
            "sweep_auto": {"bound": "alu", "frac": 0.48, "ffma_frac": 0.48,
                           "tensor_frac": 0.1}}
    bwd = {"wide_dgrad": {"bound": "tensor", "frac": 0.6, "frac_b2b": 0.7}}
    extra = {"glinear": {"bound": "tensor", "frac": 0.5}}
    out = bench.compact_rooflines(dwm, more, bwd, extra)
    assert out == {
        "dw56_s1_hbm": 0.7, "dw56_s1_b2b_hbm": 0.65, "dw1d_same_fwd_hbm": 0.2,
        "ensemble_hbm": 0.38, "ensemble_b2b_hbm": 0.39,
        "sweep_auto_alu": 0.48, "sweep_auto_ffma": 0.48, "sweep_auto_tensor": 0.1,
        "bwd_wide_dgrad_tensor": 0.6, "bwd_wide_dgrad_b2b_tensor": 0.7,
        "glinear_tensor": 0.5}
    assert bench.compact_rooflines(None, None, None) == {}
