"""Host-side pieces of bench.py that the JSON line depends on (no GPU)."""
import json

import pytest

import bench
import synth


def test_fp32_peak_from_unit_counts_and_clock():
    # 148 SMs x 128 FP32 lanes per clock x 1965 MHz
    assert bench.fp32_peak_tops(1965.0) == pytest.approx(148 * 128 * 1965e6 / 1e12)
    assert bench.fp32_peak_tops(1965.0) == pytest.approx(37.22, abs=0.01)


def test_roofline_fractions_follow_the_survey_count_and_the_fma_count():
    # the 4096 x 11008 16:32 workload (T = 300) at 3.529 ms per call, against
    # the unit-count peaks at 1965 MHz: MUFU 148 x 16, FP32 148 x 128 per clock
    params, M, T, ms = 4096 * 11008, 32, 300, 3.529
    peaks = {"fma_tops": bench.fp32_peak_tops(1965.0), "mufu_tops": bench.mufu_peak_tops(1965.0)}
    assert peaks["mufu_tops"] == pytest.approx(148 * 16 * 1965e6 / 1e12)
    r = bench.roofline_record(params, M, T, ms, peaks)
    t = ms / 1e3
    mufu = params * T * (1 + 2 / M) / (peaks["mufu_tops"] * 1e12) / t     # 318.75 ex2/lg2 per param
    fp32 = params * T * 8 / (peaks["fma_tops"] * 1e12) / t
    fma = params * T * 3 / (peaks["fma_tops"] * 1e12) / t
    assert r["frac_survey"]["mufu"] == pytest.approx(mufu) and mufu == pytest.approx(0.875, abs=0.001)
    assert r["frac_survey"]["fp32"] == pytest.approx(fp32) and fp32 == pytest.approx(0.824, abs=0.001)
    assert r["frac_fma"] == pytest.approx(fma) and fma == pytest.approx(0.309, abs=0.001)
    # the slower roofline binds: the MUFU one here, and `frac` is its fraction
    assert r["binding_pipe"] == "mufu"
    assert r["frac"] == pytest.approx(r["frac_survey"]["binding"]) and r["frac"] == pytest.approx(mufu)
    assert r["achieved"] / r["peak"] == pytest.approx(r["frac"])
    # with a slow FP32 pipe the FP32 roofline binds instead
    r2 = bench.roofline_record(params, M, T, ms, {"fma_tops": 10.0, "mufu_tops": peaks["mufu_tops"]})
    assert r2["binding_pipe"] == "fp32" and r2["frac"] == pytest.approx(r2["frac_survey"]["fp32"])


def test_clock_window_summary():
    cs = object.__new__(bench.ClockSampler)
    cs.max_mhz = 1965.0
    cs.samples = [(0.000, 1965.0, 0x0, 300.0), (0.002, 1950.0, 0x4, None), (0.004, 1965.0, 0x0, None),
                  (0.050, 900.0, 0x40, 500.0)]
    w = cs.window(0.0, 0.005)
    assert w["samples"] == 3 and w["sm_mhz"] == 1965.0 and w["sm_mhz_min"] == 1950.0
    assert w["reasons"] == ["sw_power_cap"] and w["power_w_max"] == 300.0
    assert cs.window(0.0, 0.06)["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]


def test_workload_shape_override():
    args = bench.parse_args(["--workload", "w8192x28672_bf16_laplace_32of64", "--shape", "2048x8192"])
    w = bench.workload_of(args)
    base = synth.WORKLOADS["w8192x28672_bf16_laplace_32of64"]
    assert (w.rows, w.cols) == (2048, 8192)
    assert (w.N, w.M, w.tau, w.iters, w.sweeps, w.dist) == (base.N, base.M, base.tau, base.iters, base.sweeps,
                                                            base.dist)
    with pytest.raises(SystemExit):
        bench.workload_of(bench.parse_args(["--workload", "w8192x28672_bf16_laplace_32of64", "--shape", "100x64"]))


def test_traffic_figure_only_for_todays_sources(tmp_path, monkeypatch):
    rec = {"k<bf16>": {"dram_bytes_per_launch": 123, "source_digest": bench.source_digest()},
           "old<bf16>": {"dram_bytes_per_launch": 456, "source_digest": "0" * 16}}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    real_digest = bench.source_digest()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "source_digest", lambda: real_digest)
    assert bench.profiled_traffic("k<bf16>") == 123
    assert bench.profiled_traffic("old<bf16>") is None          # counters taken on other sources
    assert bench.profiled_traffic("missing<bf16>") is None


def test_blocks_identical_counts_whole_blocks():
    torch = pytest.importorskip("torch")
    rows, cols, M = 64, 64, 32
    a = torch.zeros((rows, cols // 32), dtype=torch.int32)
    b = a.clone()
    b[5, 1] ^= 1                                              # column 32 of row 5: block (0, 1)
    b[40, 0] ^= 1 << 31                                       # column 31 of row 40: block (1, 0)
    assert bench.blocks_identical(a, b, rows, cols, M) == pytest.approx(2 / 4)
    assert bench.blocks_identical(a, a.clone(), rows, cols, M) == 1.0
