"""Host logic of bench.py on CPU: step statistics, the roofline denominator and the
dominant-GEMM roofline, and the DRAM-traffic record keyed by the kernel sources."""
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_host", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_step_stats(bench):
    st = bench.step_stats([5.0, 1.0, 3.0, 2.0, 4.0])
    assert st["median"] == 3.0 and st["mean"] == 3.0 and st["n"] == 5
    assert st["p10"] <= st["median"] <= st["p90"]
    assert st["p10"] >= 1.0 and st["p90"] <= 5.0


def test_roofline_peak_sustained_only_for_long_loops(bench):
    peak, kind = bench.roofline_peak(670.0, 1631.1, 1375.3, "measured")
    assert peak == 1375.3 and "sustained" in kind and "0.67 s" in kind
    peak, kind = bench.roofline_peak(30.0, 1631.1, 1375.3, "measured")
    assert peak == 1631.1 and "burst" in kind
    peak, kind = bench.roofline_peak(670.0, 1590.0, None, "fallback")
    assert peak == 1590.0 and "burst" in kind


def test_gemm_roofline_picks_the_largest_total_time(bench):
    from bit_quantized_mixture_nf4_b200 import workloads as wl
    w = wl.MIXTRAL
    kernels = {"gemm_gateup": {"avg_ms": 7.0, "launches": 30}, "gemm_down": {"avg_ms": 3.5, "launches": 30},
               "gemm_dgrad_down": {"avg_ms": 3.8, "launches": 30}, "gemm_dgrad_gateup": {"avg_ms": 7.2, "launches": 30}}
    roof, per = bench.gemm_roofline(w, kernels, 1375.3, "sustained", 1631.1)
    assert roof["kernel"] == "gemm_dgrad_gateup"
    flops = 4 * w.H * w.I * w.P
    assert roof["flops_per_launch"] == flops
    assert roof["achieved"] == pytest.approx(flops / 7.2e-3 / 1e12)
    assert roof["frac"] == pytest.approx(roof["achieved"] / 1375.3)
    assert roof["frac_of_burst"] == pytest.approx(roof["achieved"] / 1631.1)
    assert per["gemm_down"]["tflops"] == pytest.approx(2 * w.H * w.I * w.P / 3.5e-3 / 1e12)


def test_recorded_traffic_follows_the_kernel_sources(bench, monkeypatch):
    v = bench.recorded_traffic("gemm_gateup", "mixtral_T16384")
    assert v is None or v > 0                 # present while the record matches the sources
    assert bench.recorded_traffic("gemm_gateup", "no_such_workload") is None
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0000000000000000")
    assert bench.recorded_traffic("gemm_gateup", "mixtral_T16384") is None   # kernel changed since
