"""Host-side logic of bench.py (no GPU): the clock record that decides
whether a timed run is kept, the gate that reports committed DRAM traffic
only for the kernel sources it was captured with, and the workload names."""
import json

import pytest

import bench

IDLE = "0, 1965, 1965, 150.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n"
CAPPED = "0, 1447, 1965, 998.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n"
THERMAL = "0, 1200, 1965, 700.0, 0x0000000000000040, Not Active, Active, Not Active, Not Active\n"


def test_clock_summary_median_and_reasons():
    s = bench.ClockSampler.summarize([IDLE, CAPPED, CAPPED, "garbage\n", "0, N/A, 1965, 1, a, b, c, d, e\n"])
    assert s["samples"] == 3                    # the two malformed lines are skipped
    assert s["sm_mhz"] == 1447.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_summary_reports_a_rejecting_reason():
    s = bench.ClockSampler.summarize([IDLE, THERMAL])
    assert "hw_thermal_slowdown" in s["reasons"] and "sw_power_cap" not in s["reasons"]


def test_clock_summary_without_samples():
    assert bench.ClockSampler.summarize([]) == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_traffic_only_for_the_captured_sources(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    with open(tmp_path / "profiles" / "traffic.json", "w") as f:
        json.dump({"csrc_sha256_16": "aaaa", "ffn": {"fp8_gemm_up": 123}}, f)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "csrc_hash", lambda: "aaaa")
    assert bench.load_traffic("fp8_gemm_up", "ffn") == 123
    assert bench.load_traffic("fp8_gemm_up", "moe") is None          # no capture for that workload
    assert bench.load_traffic("quant_rows_up", "ffn") is None        # nor for that kernel
    monkeypatch.setattr(bench, "csrc_hash", lambda: "bbbb")          # the kernels changed since
    assert bench.load_traffic("fp8_gemm_up", "ffn") is None


def test_committed_traffic_covers_the_bench_workloads():
    with open(bench.os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        t = json.load(f)
    assert len(t["csrc_sha256_16"]) == 16
    for workload in ("ffn", "moe", "moe_tokens", "sweep_m128"):
        assert t[workload] and all(isinstance(v, int) and v > 0 for v in t[workload].values()), workload


def test_csrc_hash_is_stable():
    assert bench.csrc_hash() == bench.csrc_hash() and len(bench.csrc_hash()) == 16


@pytest.mark.parametrize("name,kind,n", [("tiny", "dense", 1), ("sweep_m8", "dense", 1)])
def test_workload_spec_shapes(name, kind, n):
    desc, k, tensors = bench.workload_spec(name)
    assert k == kind and len(tensors) == n and desc
    X, W = tensors[0]
    assert X.shape[1] == W.shape[1]


def test_unknown_workload_is_rejected():
    with pytest.raises(SystemExit):
        bench.workload_spec("no_such_workload")
