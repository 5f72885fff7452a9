"""Host-side pieces of bench.py that the JSON line depends on (no GPU)."""
import json

import pytest

import bench
import synth


def test_fp32_peak_from_unit_counts_and_clock():
    # 148 SMs x 128 FP32 lanes per clock x 1965 MHz
    assert bench.fp32_peak_tops(1965.0) == pytest.approx(148 * 128 * 1965e6 / 1e12)
    assert bench.fp32_peak_tops(1965.0) == pytest.approx(37.22, abs=0.01)


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
