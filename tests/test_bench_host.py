"""Host logic of bench.py that needs no GPU: the source-hash gate on captured DRAM
traffic, the peaks fallback, the clock summary and the algorithmic flop count the
solve's roofline divides by."""
import hashlib
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_traffic_is_reported_only_for_the_captured_source(monkeypatch):
    # a committed file stands in for a kernel source; nothing is written
    src = "include/gka.h"
    with open(os.path.join(ROOT, src), "rb") as f:
        digest = hashlib.sha1(f.read()).hexdigest()
    monkeypatch.setitem(bench.TRAFFIC, "kern",
                        {"bytes": 123.0e6, "workload": "wl", "src": src, "sha1": digest})
    assert bench.traffic_of("kern", "wl") == 123.0e6
    # another workload, or a kernel without a capture: no figure
    assert bench.traffic_of("kern", "other") is None
    assert bench.traffic_of("no_such_kernel", "wl") is None
    # the source changed since the capture: no figure
    monkeypatch.setitem(bench.TRAFFIC, "kern",
                        {"bytes": 123.0e6, "workload": "wl", "src": src, "sha1": "0" * 40})
    assert bench.traffic_of("kern", "wl") is None
    # the source is gone: no figure
    monkeypatch.setitem(bench.TRAFFIC, "kern",
                        {"bytes": 123.0e6, "workload": "wl", "src": "no/such/file.cuh",
                         "sha1": digest})
    assert bench.traffic_of("kern", "wl") is None


def test_traffic_table_names_existing_sources():
    for name, t in bench.TRAFFIC.items():
        assert os.path.exists(os.path.join(ROOT, t["src"])), name
        assert len(t["sha1"]) == 40 and t["bytes"] > 0, name


def test_peaks_fall_back_without_measured_file(monkeypatch):
    # a committed folder without a measured-peaks file
    monkeypatch.setattr(bench, "ROOT", os.path.join(ROOT, "tests", "golden"))
    p = bench.load_peaks()
    assert p["_source"] == "fallback"
    assert p["hbm_gbs"] == bench.FALLBACK_PEAKS["hbm_gbs"]
    monkeypatch.setattr(bench, "ROOT", ROOT)
    if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")):
        p = bench.load_peaks()
        assert p["_source"] == "measured" and p["hbm_gbs"] > 0


def test_solve_flops_per_head_token():
    # r rounds of three products per token at C = 64, D = 128 (K X^T: 2CD,
    # H_s X^T: 2D^2, K^T P^T: 2CD): the r - 1 Chebyshev products plus the readout
    D, C, r = 128, 64, 20
    ch, out, upd, nrm = bench.flops_per_head_token(D, C, r)
    assert ch + out == r * (2 * C * D + 2 * D * D + 2 * D * C) == 1_310_720
    assert upd == 4 * D * D
    assert nrm == 2 * D * D + 2 * C * D + 2 * C * C
    # the tensor-core solve also forms every token's norm (fused), so its own count
    # is Chebyshev + readout + norm; the CUDA-core solve leaves the norm to its kernel
    assert bench.kernel_flops_per_head_token("chunk_solve_tc", D, C, r) == 1_310_720 + 57_344
    assert bench.kernel_flops_per_head_token("chunk_solve", D, C, r) == 1_310_720
    assert bench.kernel_flops_per_head_token("chunk_norm", D, C, r) == nrm
    assert bench.kernel_flops_per_head_token("state_pass_tc", D, C, r) == upd
    assert bench.kernel_flops_per_head_token("state_scan", D, C, r) == 0


def test_clock_summary_flags_throttle_reasons():
    s = bench.ClockSampler(0)
    assert s.summary()["reasons"] == ["unsampled"]
    s.max_mhz = 1965.0
    s.samples = [(1965.0, 0), (1850.0, 0x4), (1900.0, 0)]
    out = s.summary()
    assert out["sm_mhz"] == 1900.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"] and out["samples"] == 3
    s.samples.append((1200.0, 0x40 | 0x8))
    assert s.summary()["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_power_cap"]


@pytest.mark.parametrize("D,C", [(128, 32), (64, 16)])
def test_backward_flops_are_per_kernel(D, C):
    fl = bench.bwd_flops_per_head_token(D, C, 20)
    assert fl["bwd_rows"] == 7 * 2 * D * D
    assert fl["bwd_delta"] == 3 * 2 * D * D
    assert fl["bwd_solve"] == (2 * D * D + 4 * C * D) + fl["chunk_solve"]


def test_forward_roofline_counts_the_solve_with_its_norm():
    from test_ridge_regression_b200.inputs import WORKLOADS
    w = WORKLOADS["bf16_b8h8t2048d128"]
    peaks = {"bf16_tflops": 1000.0, "sm_max_mhz": 1965.0, "_source": "test"}
    # 20 steps, the solve 0.5 ms per step, the state pass 0.1 ms: the solve dominates
    kt = {"chunk_solve_tc": (10.0, 20), "state_pass_tc": (2.0, 20)}
    roof = bench.forward_roofline(w, kt, 20, 0.65, peaks)
    head_tok = w.B * w.H * w.T
    flops = (1_310_720 + 57_344) * head_tok
    assert roof["kernel"] == "chunk_solve_tc" and roof["bound"] == "tensor"
    assert roof["algorithmic_per_step"] == flops
    assert abs(roof["achieved"] - flops / 0.5e-3 / 1e12) < 1e-6
    assert abs(roof["frac"] - roof["achieved"] / 1000.0) < 1e-12
    whole = 1_433_600 * head_tok
    assert abs(roof["step_frac_of_bf16_peak"] - whole / 0.65e-3 / 1e12 / 1000.0) < 1e-12
