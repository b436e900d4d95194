"""bench.py host logic that needs no GPU: the roofline's traffic figure is
reported only while the kernel sources are the ones it was taken on, the peaks come from the measured file, and the clock
sampler decodes throttle reasons from a fake NVML (it only reads)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_traffic_is_reported_only_for_the_sources_it_was_taken_on(monkeypatch):
    monkeypatch.setattr(bench, "GEMM_TRAFFIC", {"bytes_per_launch": 123456789, "workload": "w",
                                                "sources_sha256": bench.gemm_sources_sha256()})
    assert bench.gemm_traffic() == (123456789, "w")
    monkeypatch.setattr(bench, "gemm_sources_sha256", lambda: "0" * 64)
    assert bench.gemm_traffic() == (None, None)


def test_the_committed_traffic_figure_is_consistent():
    t = bench.GEMM_TRAFFIC
    if t["sources_sha256"] is not None:
        assert len(t["sources_sha256"]) == 64 and 1e8 < t["bytes_per_launch"] < 1e10 and t["workload"]


def test_the_source_hash_covers_the_gemm_sources():
    h1 = bench.gemm_sources_sha256()
    assert len(h1) == 64 and h1 == bench.gemm_sources_sha256()
    assert "grouped_gemm.cu" in bench.GEMM_SOURCES and "ptx.cuh" in bench.GEMM_SOURCES


def test_peaks_come_from_the_measured_file():
    pk = bench.peaks()
    if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")):
        assert pk["src"] == "measured" and pk["hbm_gbs"] > 1000 and pk["bf16"] > 100
    else:
        assert pk["src"] == "fallback"


class _FakeNVML:
    nvmlClocksThrottleReasonSwPowerCap = 0x4
    nvmlClocksThrottleReasonHwSlowdown = 0x8
    nvmlClocksThrottleReasonSwThermalSlowdown = 0x20
    nvmlClocksThrottleReasonHwThermalSlowdown = 0x40


def test_clock_reasons_are_decoded_from_the_mask():
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.nv = _FakeNVML()
    assert s._reason_names(0x4) == {"sw_power_cap"}
    assert s._reason_names(0x4 | 0x40) == {"sw_power_cap", "hw_thermal_slowdown"}
    assert s._reason_names(0x0) == set()
    assert bench.ClockSampler.BAD == {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}


def test_summary_reports_the_median_clock():
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.samples, s.reasons, s.max_mhz = [1500, 1700, 1650], {"sw_power_cap"}, 1965
    out = s.summary()
    assert out == {"sm_mhz": 1650, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"], "samples": 3}


def test_system_info_reads_what_it_can():
    info = bench.system_info(0)
    assert set(info) == {"gpu", "driver", "cuda", "torch", "host_cores"}
    assert info["torch"] and info["host_cores"] >= 1


def test_both_arms_share_one_config():
    from mxfp8_grouped_gemm_quantize_b200 import workloads as wl
    w = wl.ds_v3_16b()
    c = bench.workload_config(w, "dual", 1)
    assert c["workload"] == "ds-v3-16b-like MoE layer" and c["routed_rows"] == 49152 and c["experts"] == 64
    assert c["layers"] == [{"name": "gate_up", "N": 2816, "K": 2048}, {"name": "down", "N": 2048, "K": 1408}]
    assert c["parallelism"] == "replica x1"


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` (the oracle on the host cores) prints one
    JSON line with the contract's keys and the same config as our arm."""
    import json
    import subprocess
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"],
                       cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    from mxfp8_grouped_gemm_quantize_b200 import workloads as wl
    assert d["config"] == bench.workload_config(wl.ds_v3_671b(), "dual", 1)
    assert d["metric"] == bench.METRIC and d["unit"] == bench.UNIT


def test_the_headline_is_the_671b_like_layer():
    from mxfp8_grouped_gemm_quantize_b200 import workloads as wl
    assert bench.WORKLOAD == "ds-v3-671b"
    c = bench.workload_config(wl.ds_v3_671b(), "dual", 1)
    assert c["workload"] == "ds-v3-671b-like MoE layer" and c["routed_rows"] == 16384 and c["experts"] == 32
    assert c["layers"] == [{"name": "gate_up", "N": 4096, "K": 7168}, {"name": "down", "N": 7168, "K": 2048}]
    assert "Zipf" in c["routing"]


def test_in_step_kernels_are_held_to_the_sustained_peak_in_long_runs():
    pk = {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sust": 1400.0, "src": "fallback"}
    assert bench.step_peak(pk, 1300.0) == (2800.0, "sustained")
    assert bench.step_peak(pk, 80.0) == (3180.0, "burst")
    assert bench.step_peak(dict(pk, bf16_sust=None), 1300.0) == (3180.0, "burst")
