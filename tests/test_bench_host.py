"""bench.py's host-side logic on CPU: the roofline object (bound, peak
choice, fractions), the clock-sample summary, and the guard that drops DRAM
traffic figures once a kernel's sources have changed since their capture."""
import json

import pytest

import bench

PEAKS = ({"bf16_tflops": 1700.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6400.0}, "measured")


def test_roofline_tensor_bound_takes_burst_or_sustained_peak():
    flops = 2.0 * 8192 ** 3
    alg = (2 * 8192 * 8192 + 8192 * 8192) * 2
    ms = flops / 1374e12 * 1e3  # 1374 TFLOP/s
    long_run = bench._roofline(flops, alg, ms, 800.0, True, "bf16", PEAKS)
    assert long_run["bound"] == "tensor" and long_run["unit"] == "TFLOP/s"
    assert long_run["peak"] == 1400.0 and "sustained" in long_run["peak_source"]
    assert long_run["frac"] == pytest.approx(1374 / 1400, abs=1e-4)
    assert long_run["frac_of_burst"] == pytest.approx(1374 / 1700, abs=1e-4)
    # short, or L2-flushed between steps: the burst figure
    for total_ms, b2b in ((100.0, True), (800.0, False)):
        r = bench._roofline(flops, alg, ms, total_ms, b2b, "f16", PEAKS)
        assert r["peak"] == 1700.0 and "(burst)" in r["peak_source"]
        assert "fp16 has the same dense rate" in r["peak_source"]
    assert long_run["bound_times_us"]["tensor"] == pytest.approx(flops / 1400e12 * 1e6, abs=0.01)


def test_roofline_hbm_bound_reports_bytes_per_second():
    flops = 2.0 * 16 * 8192 * 8192
    alg = (16 * 8192 + 8192 * 8192 + 16 * 8192) * 2
    ms = 0.037
    r = bench._roofline(flops, alg, ms, 7.4, True, "f16", PEAKS)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == 6400.0
    assert r["achieved"] == pytest.approx(alg / (ms * 1e-3) / 1e9, abs=0.1)
    assert r["frac"] == pytest.approx(r["achieved"] / 6400.0, abs=1e-4)
    assert r["bound_times_us"]["hbm"] > r["bound_times_us"]["tensor"]


def test_roofline_without_measured_peaks_uses_the_fallback():
    r = bench._roofline(2.0 * 4096 ** 3, 100e6, 0.1, 20.0, False, "bf16",
                        (dict(bench.FALLBACK_PEAKS), "fallback"))
    assert r["peak"] == bench.FALLBACK_PEAKS["bf16_tflops"]
    assert r["peak_source"].startswith("fallback")


def test_clock_summary_median_and_reasons():
    c = bench.ClockSampler(0)
    c.lines = [
        "0, 1965, 1965, 500.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1400, 1965, 999.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1300, 1965, 1000.2, 0x4, Not Active, Not Active, Not Active, Active",
        "garbled line",
        "0, N/A, 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    s = c.summary()
    assert s["sm_mhz"] == 1400.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 3
    c.lines.append("0, 1200, 1965, 900, 0x40, Not Active, Active, Not Active, Not Active")
    assert c.summary()["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]


def test_traffic_dropped_once_a_kernel_source_changes(tmp_path, monkeypatch):
    csrc = tmp_path / "dense_gemm_16_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "common.cuh").write_text("// shared\n")
    (csrc / "kernel.cu").write_text("// kernel v1\n")
    (csrc / "other.cu").write_text("// another kernel\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    srcs = ["common.cuh", "kernel.cu"]
    entry = {"sources": srcs, "source_sha": bench._source_sha(srcs),
             "dram_bytes_per_launch": 12345}
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps({"w": entry}))
    assert bench._traffic("w") == 12345
    assert bench._traffic("unknown") is None
    (csrc / "other.cu").write_text("// another kernel, edited\n")  # not this kernel's source
    assert bench._traffic("w") == 12345
    (csrc / "kernel.cu").write_text("// kernel v2\n")
    assert bench._traffic("w") is None


def test_reference_arm_line_matches_the_contract(capsys):
    """`bench.py --impl reference` (the oracle timed on the host cores) prints
    one JSON line with our arm's metric, unit and workload config."""
    import workloads
    bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3",
                "--workload", "square256_f16"])
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["higher_is_better"] is True and d["value"] > 0
    assert d["config"] == bench._workload_config(workloads.get("square256_f16"), 1)
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
