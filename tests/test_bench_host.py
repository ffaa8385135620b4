"""The benchmark's host-side logic without a GPU: workload tables, the metric
and roofline bookkeeping, the ncu-summary lookup, and the reference arm (the
oracle on the host cores) printing its JSON line."""
import io
import json
import os
import sys
from contextlib import redirect_stdout

import numpy as np
import pytest

import bench
import workloads


def test_workload_metrics():
    assert bench.workload_meta("decode") == ("FP8 GEMM HBM bandwidth (M<=128)", "GB/s", "hbm")
    assert bench.workload_meta("prefill")[1:] == ("TFLOP/s", "tensor")
    assert bench.workload_meta("bf16-decode") == ("BF16 GEMM HBM bandwidth (M<=128)", "GB/s", "hbm")
    assert bench.workload_meta("bf16-prefill") == ("BF16 GEMM TFLOPS", "TFLOP/s", "tensor")
    assert bench.is_bf16("bf16-decode") and not bench.is_bf16("decode")
    assert bench.profile_name("decode") == "fp8_gemm_decode"
    assert bench.profile_name("bf16-prefill") == "bf16_gemm_prefill"


def test_step_units_and_roofline_on_the_smoke_step():
    items = bench.build_workload("smoke")
    (kind, p), = items
    M, N, K = workloads.SMOKE_SHAPE
    assert kind == "dense" and (p.M, p.N, p.K) == (M, N, K)
    # bytes: A + sfa + B + sfb + D(bf16)
    want = M * K + 4 * M * K // 128 + N * K + 4 * (-(-N // 128)) * K // 128 + 2 * M * N
    assert bench.step_units(items, "GB/s") == want
    assert bench.step_units(items, "TFLOP/s") == 2 * M * N * K
    r = bench.roofline_terms(items, ms=1e-3, hbm_gbs=1000.0, fp8_tflops=1000.0)
    assert r["bound"] == "hbm"
    assert r["t_roof_s"] == pytest.approx(max(want / 1e12, 2 * M * N * K / 1e15))
    assert r["frac_time"] == pytest.approx(r["t_roof_s"] / 1e-6)


def test_launches_per_step_count_the_tail_launches():
    """gpu_launches counts every kernel launch of a step: one per GEMM, plus
    the split-off last wave of a dense GEMM (the library's own plan)."""
    assert bench.step_launches(bench.build_workload("decode")) == 6
    # 4096 x 7168 x 16384 splits its last wave into one tail launch
    assert bench.step_launches(bench.build_workload("prefill")) == 5
    assert bench.step_launches(bench.build_workload("bf16-prefill")) == 5
    assert bench.step_launches(bench.build_workload("masked")) == 1


def test_bf16_problem_units():
    p = workloads.bf16_dense_problem(64, 256, 512, seed=0)
    assert p.a.dtype == np.uint16 and p.a.shape == (64, 512) and p.b.shape == (256, 512)
    assert p.bytes() == 2 * 64 * 512 + 2 * 256 * 512 + 2 * 64 * 256
    items = [("bf16_dense", p)]
    # a BF16 step against the BF16 peak: the tensor term is twice the E4M3 one
    r8 = bench.roofline_terms(items, 1.0, 1e9, 2000.0)
    r16 = bench.roofline_terms(items, 1.0, 1e9, 1000.0, bench.SPEC_BF16_TFLOPS)
    assert r16["t_roof_s"] == pytest.approx(2 * r8["t_roof_s"])


def test_traffic_lookup_checks_the_source_hash(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "abc123")
    assert bench.profiled_traffic("decode") is None                 # no summary
    (prof / "fp8_gemm_decode_traffic.md").write_text(
        "# x\n\ntraffic_bytes_per_launch: 1234\nkernel_source_hash: abc123\n")
    assert bench.profiled_traffic("decode") == 1234
    (prof / "fp8_gemm_decode_traffic.md").write_text(
        "traffic_bytes_per_launch: 1234\nkernel_source_hash: other\n")
    assert bench.profiled_traffic("decode") is None                 # other sources


def test_the_committed_summaries_name_a_source_hash():
    for w in ("decode", "prefill", "contiguous", "masked"):
        path = os.path.join(bench.ROOT, "profiles", f"{bench.profile_name(w)}_traffic.md")
        text = open(path).read()
        assert "traffic_bytes_per_launch:" in text and "kernel_source_hash:" in text


@pytest.mark.parametrize("workload", ["smoke"])
def test_reference_arm_prints_one_json_line(workload, monkeypatch):
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--workload", workload,
                                      "--steps", "3", "--warmup", "3"])
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.main()
    lines = [l for l in buf.getvalue().splitlines() if l.strip()]
    assert len(lines) == 1
    res = json.loads(lines[0])
    assert res["impl"] == "reference" and res["unit"] == "GB/s" and res["value"] > 0
    assert res["cpu_baseline"]["kind"] == "oracle" and res["cpu_baseline"]["cores"] >= 1
    assert res["e2e"]["h2d_bytes_per_step"] == 0 and res["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_do_nothing(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--workload", "smoke",
                                      "--steps", "3", "--warmup", "3"])
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.main()
    assert buf.getvalue().strip() == ""


def test_warmup_below_three_is_refused(monkeypatch):
    monkeypatch.setattr(sys, "argv", ["bench.py", "--warmup", "2"])
    with pytest.raises(SystemExit):
        bench.main()


def test_clock_summary_skips_idle_samples_and_reads_reasons():
    """Samples taken while the GPU was idle (bit 0 of the active-reasons mask)
    are left out of the median; throttle reasons are collected by name."""
    c = bench.ClockSampler(0)
    c.lines = [
        "1072, 1965, 100.0, 0x0000000000000001, Not Active, Not Active, Not Active, Not Active",
        "1965, 1965, 700.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "1900, 1965, 990.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "1965, 1965, 710.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
    ]
    s = c.summary()
    assert s["samples"] == 3 and s["idle_samples"] == 1
    assert s["sm_mhz"] == 1965.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]


def test_long_timed_regions_use_the_sustained_tensor_peak():
    """20 prefill steps (15 ms) are held against the burst E4M3 peak; 2000
    steps (1.5 s, the power cap acting) against the sustained one."""
    items = bench.build_workload("prefill")
    t = {"items": items, "ms": 0.77, "unit": "TFLOP/s", "metric": "m", "R": 2, "flush_note": "",
         "preload": False, "clocks": {}, "kernel_ms": [], "ms_alt": None}
    short = bench.workload_record("prefill", t, 1, 20, 5)["roofline"]
    long = bench.workload_record("prefill", t, 1, 2000, 5)["roofline"]
    assert "sustained" not in short["peak_source"] and "sustained" in long["peak_source"]
    assert long["peak"] < short["peak"]
    assert long["frac"] == pytest.approx(short["frac"] * short["peak"] / long["peak"], rel=1e-3)
