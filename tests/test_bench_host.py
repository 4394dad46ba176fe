"""Host-side logic of bench.py (no GPU): FLOP and byte accounting, the traffic record's
validity check, the CLI's warm-up rule and the parsing of sampled clocks."""
import json

import pytest

import bench


def test_gemm_flops_per_row_counts_every_projection():
    H, KV, F, V = 4096, 1024, 12288, 151936
    expect = 2 * (H * H + H * KV + H * KV + H * H + H * 2 * F + F * H + H * V)
    assert bench.gemm_flops_per_row() == expect
    assert abs(expect / 1e9 - 1.6305) < 1e-4


def test_row_op_bytes_are_algorithmic():
    b = bench.row_op_bytes_per_row()
    assert b["log_softmax"] == 6 * 151936  # bf16 read once, fp32 written once
    assert b["mean"] == 4 * 151936 + 4
    assert b["rms1"] == 4 * 4096


def test_traffic_record_is_used_only_for_its_source_case_and_rows(tmp_path, monkeypatch):
    rec = {"gemm_source_sha": bench.gemm_source_sha(), "rows": 1024, "kernel_case": "gemm_lm_head",
           "dram_bytes_per_launch": 123456789}
    path = tmp_path / "traffic.json"
    path.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(path))
    assert bench.measured_traffic(1024, "gemm_lm_head") == 123456789
    assert bench.measured_traffic(2048, "gemm_lm_head") is None
    assert bench.measured_traffic(1024, "gemm_qo_m256") is None
    rec["gemm_source_sha"] = "0" * 16  # captured on another kernel source
    path.write_text(json.dumps(rec))
    assert bench.measured_traffic(1024, "gemm_lm_head") is None
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "missing.json"))
    assert bench.measured_traffic(1024, "gemm_lm_head") is None


def test_cli_refuses_fewer_than_three_warmup_steps(monkeypatch):
    monkeypatch.setattr("sys.argv", ["bench.py", "--warmup", "2"])
    with pytest.raises(SystemExit):
        bench.main()


class _FakeSmi:
    def __init__(self, text):
        self.text = text

    def terminate(self):
        pass

    def communicate(self, timeout=None):
        return self.text, ""


def test_clock_sampler_reports_median_and_active_reasons():
    t = "2026/12/03 10:00:00.{:03d}"
    lines = [t.format(100) + ", 0, 1800, 1965, 950.0, 0x4, Not Active, Not Active, Not Active, Active",
             t.format(200) + ", 0, 1700, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
             t.format(300) + ", 0, 1900, 1965, 900.0, 0x0, Not Active, Not Active, Not Active, Not Active",
             "garbled line"]
    s = bench.ClockSampler(0)
    s.proc = _FakeSmi("\n".join(lines))
    out = s.stop()
    assert out["sm_mhz"] == 1800 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"] and out["samples"] == 3
    s.proc = _FakeSmi(t.format(0) + ", 0, 900, 1965, 500.0, 0x8, Active, Not Active, Not Active, Not Active")
    assert s.stop()["reasons"] == ["hw_slowdown"]


def test_clock_sampler_keeps_the_samples_of_the_timed_region():
    """Samples before the timed region (an idle GPU at its maximum clock) do not count."""
    from datetime import datetime
    t = "2026/12/03 10:00:0{}.000"
    lines = [t.format(0) + ", 0, 1965, 1965, 150.0, 0x0, Not Active, Not Active, Not Active, Not Active",
             t.format(1) + ", 0, 1965, 1965, 160.0, 0x0, Not Active, Not Active, Not Active, Not Active",
             t.format(2) + ", 0, 1650, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
             t.format(3) + ", 0, 1700, 1965, 995.0, 0x4, Not Active, Not Active, Not Active, Active",
             t.format(4) + ", 0, 1680, 1965, 985.0, 0x4, Not Active, Not Active, Not Active, Active"]
    at = [datetime.strptime(t.format(i), "%Y/%m/%d %H:%M:%S.%f").timestamp() for i in range(5)]
    s = bench.ClockSampler(0)
    s.proc = _FakeSmi("\n".join(lines))
    out = s.stop((at[2] - 0.5, at[4] + 0.5))
    assert out["sm_mhz"] == 1680 and out["samples"] == 3 and out["window"] == "timed region"
    assert out["reasons"] == ["sw_power_cap"]
    s.proc = _FakeSmi("\n".join(lines))
    assert s.stop((at[4] + 10, at[4] + 11))["window"] == "whole sampling run"  # nothing inside


def test_roofline_point_takes_the_larger_bound():
    """The roofline time of a launch is the larger of its FLOPs at the tensor peak and its
    algorithmic bytes at the HBM peak; the fraction is that time over the measured one."""
    peaks = {"bf16_tflops": 1000.0, "hbm_gbs": 5000.0}
    # 2 TFLOP at 1000 TFLOP/s = 2 ms; 1 GB at 5000 GB/s = 0.2 ms: tensor-bound
    r = bench.roofline_point(2e12, 1e9, 4000.0, peaks)
    assert r == {"bound": "tensor", "roofline_frac": 0.5}
    # 1 GFLOP = 1 us of tensor time; 50 MB = 10 us of HBM time: HBM-bound, measured 20 us
    r = bench.roofline_point(1e9, 50e6, 20.0, peaks)
    assert r == {"bound": "hbm", "roofline_frac": 0.5}


def test_sweep_lists_are_distinct():
    """The extended sweep covers M = 1..2048 with the ragged points 3, 77 and 1000; the JSON
    line's metric sweep keeps its own five points."""
    assert bench.SWEEP_M == [1, 2, 3, 4, 8, 16, 32, 64, 77, 128, 256, 512, 1000, 1024, 2048]
    assert bench.METRIC_SWEEP_M == [1, 64, 256, 1024, 2048]
