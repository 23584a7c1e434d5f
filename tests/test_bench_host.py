"""Host-side logic of bench.py on the CPU: the clock summary (with a fake NVML), the
recorded-traffic lookup keyed by the kernel sources, the peaks file, the plan's
launch count and the argument defaults."""
import json
import os
import sys
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_clock_summary_keeps_the_window_and_reasons():
    fake = types.SimpleNamespace(nvmlClocksEventReasonHwSlowdown=1,
                                 nvmlClocksEventReasonHwThermalSlowdown=2,
                                 nvmlClocksEventReasonSwThermalSlowdown=4,
                                 nvmlClocksEventReasonSwPowerCap=8,
                                 nvmlClocksEventReasonHwPowerBrakeSlowdown=16)
    c = bench.ClockSampler(0)
    c._nvml = fake
    c.max_mhz = 1965
    c.samples = [(0.5, 1000.0, 1, 100.0),            # before the window: ignored
                 (1.0, 1965.0, 0, 500.0), (1.1, 1900.0, 8, 900.0), (1.2, 1800.0, 0, 700.0),
                 (3.0, 500.0, 2, 100.0)]             # after the window: ignored
    c.mark(1.0, 2.0)
    out = c.stop()
    assert out["sm_mhz"] == 1900.0 and out["sm_mhz_min"] == 1800.0
    assert out["reasons"] == ["sw_power_cap"]
    assert out["samples"] == 3 and out["power_w_max"] == 900.0 and out["sm_max_mhz"] == 1965


def test_recorded_traffic_is_tied_to_the_kernel_sources():
    with open(bench.TRAFFIC_FILE) as f:
        rows = json.load(f)
    sha = bench.kernel_sources_sha()
    for r in rows:
        got = bench.measured_traffic(r["kernel"], r["workload"])
        assert got == (r["dram_bytes_per_launch"] if r["source_sha"] == sha else None)
    assert bench.measured_traffic("gemm1_swiglu", "no_such_workload") is None


def test_peaks_file_or_fallback():
    p, kind = bench.peaks()
    assert kind in ("measured", "fallback")
    assert p["hbm_gbs"] > 1000 and p["bf16_tflops"] > 100


def test_plan_launch_count():
    # one launch while the rows fit one chunk of 16 warps x 32 rows, two beyond
    assert bench.plan_launches(512, 148) == 1
    assert bench.plan_launches(513, 148) == 2
    assert bench.plan_launches(8192, 148) == 2
    assert bench.plan_launches(1, 148) == 1


def test_default_arguments():
    a = bench.parse_args([])
    # the headline is the largest single-GPU workload; every other one gets a record
    assert (a.gpus, a.steps, a.warmup, a.impl, a.workload) == (1, 20, 5, "ours", "phi35")
    assert a.warmup >= 3 and a.side_warmup >= 3
    from grouped_gemm_plan_b200 import workload as W
    flops = {n: W.WORKLOADS[n].flops() for n in W.WORKLOADS if not n.endswith("_prof")}
    assert max(flops, key=flops.get) == a.workload
    assert set(a.side.split(",")) | {a.workload} == set(flops)


def test_compact_rounding():
    assert bench._r(1234567.0) == 1235000.0
    assert bench._r(0.93817, 3) == 0.938
    assert bench._r(0.0) == 0.0 and bench._r(None) is None


def test_reference_arm_line(capsys, monkeypatch):
    # the CPU oracle arm on the tiny workload: measured per-step time, the same
    # config object as the GPU arm, the CPU model recorded
    monkeypatch.delenv("RANK", raising=False)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    args = bench.parse_args(["--impl", "reference", "--workload", "tiny", "--steps", "3",
                             "--warmup", "1", "--cpu-seconds", "1.5"])
    assert bench.run_reference(args) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    from grouped_gemm_plan_b200 import workload as W
    assert line["impl"] == "reference" and line["steps"] == 3
    assert line["config"] == bench.workload_config(W.WORKLOADS["tiny"], 1)
    per_step_s = line["ms_per_step"] / 1e3
    assert 0.0 < per_step_s < 5.0                      # measured, not extrapolated
    assert abs(line["tokens_per_step"] / per_step_s - line["value"]) <= 0.05 * line["value"]
    assert line["ms_per_full_batch_extrapolated"] >= line["ms_per_step"] * 0.99
    assert line["cpu_baseline"]["cpu_model"] and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0
