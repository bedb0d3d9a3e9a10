"""Host-side pieces of the benchmark that need no GPU: the clock-sample
parser, the validity check of the committed DRAM-traffic record, the peak
fallback, and the algorithmic byte and flop counts."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from lm_head_loss_junction_b200 import workloads as wl  # noqa: E402


def test_clock_summary_takes_the_median_and_collects_reasons():
    cs = bench.ClockSampler(0)
    cs.lines = [
        "0, 1200, 1965, 950.1, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1300, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1250, 1965, 970.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ]
    s = cs.summary()
    assert s["sm_mhz"] == 1250 and s["sm_max_mhz"] == 1965 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"]
    cs.lines = ["0, 900, 1965, 500, 0x0, Active, Not Active, Active, Not Active"]
    assert bench.ClockSampler.summary(cs)["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    cs.lines = []
    assert cs.summary()["sm_mhz"] is None


def test_traffic_record_is_used_only_for_the_captured_source(tmp_path, monkeypatch):
    import hashlib
    cfg = wl.CONFIGS["main3"]
    fake_root = tmp_path / "repo"
    (fake_root / "profiles").mkdir(parents=True)
    src_dir = fake_root / "lm_head_loss_junction_b200" / "csrc"
    src_dir.mkdir(parents=True)
    text = "// a kernel source\n"
    (src_dir / "loss_tc.cu").write_text(text)
    rec = {"source": "lm_head_loss_junction_b200/csrc/loss_tc.cu",
           "source_sha256_16": hashlib.sha256(text.encode()).hexdigest()[:16],
           "dram_bytes_read_per_launch": 3.0e9, "dram_bytes_write_per_launch": 0.5e8}
    (fake_root / "profiles" / "traffic_loss_tile_stats_main3_T8192.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(fake_root))
    assert bench.measured_traffic(cfg) == pytest.approx(3.05e9)          # the captured source
    assert bench.measured_traffic(wl.CONFIGS["proxy2"]) is None          # another workload
    (src_dir / "loss_tc.cu").write_text(text + "// edited\n")
    assert bench.measured_traffic(cfg) is None                            # the source changed since
    (fake_root / "profiles" / "traffic_loss_tile_stats_main3_T8192.json").unlink()
    assert bench.measured_traffic(cfg) is None                            # no record at all


def test_peaks_fall_back_when_the_file_is_missing(monkeypatch, tmp_path):
    monkeypatch.setattr(bench, "PEAKS_FILE", str(tmp_path / "missing.json"))
    peaks, kind = bench.load_peaks()
    assert kind == "fallback" and peaks["hbm_gbs"] > 0 and peaks["bf16_tflops"] > 0


def test_algorithmic_counts_of_the_main_suite():
    c = wl.CONFIGS["main3"]
    step = object.__new__(bench.Step)          # the counts need only the config
    step.cfg = c
    fwd, bwd = step.junction_bytes()
    # per token: forward (D + delta + D_next) * 2 + 8 bytes, backward rows (D_next + 2D + 2 delta) * 2 + 8
    assert fwd == c.T * ((1024 + 1280 + 2304) * 2 + 8 + (2304 + 2048 + 4352) * 2 + 8)
    rows = c.T * ((2304 + 2 * 1024 + 2 * 1280) * 2 + 8 + (4352 + 2 * 2304 + 2 * 2048) * 2 + 8)
    # plus the fp32 tables written once (V x delta x 4) and g_e, coef read again (T x (delta * 2 + 4))
    tables = c.V * (1280 + 2048) * 4 + c.T * ((1280 + 2048) * 2 + 8)
    assert bwd == rows + tables
    assert 1.0e9 < bwd < 1.1e9                 # about 1.04 GB per step at T = 8192
    assert step.loss_flops_algorithmic() == 6.0 * c.T * c.V * (1024 + 2304 + 4352)
    assert step.loss_flops_executed() == 8.0 * c.T * c.V * (1024 + 2304 + 4352)
