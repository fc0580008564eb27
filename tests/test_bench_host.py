"""Host logic of bench.py on CPU: the clock sampler's reading of nvidia-smi
samples, the lookup of recorded DRAM traffic, and the weak-scaling value."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _sampler(samples):
    s = object.__new__(bench.ClockSampler)       # no nvidia-smi process
    s.proc = None
    s.samples = samples
    return s


def test_clock_sampler_takes_the_median_of_the_timed_window_and_its_reasons():
    idle = ["600", "1965", "150.0", "Not Active", "Not Active", "Not Active", "Not Active"]
    busy = lambda mhz, cap: [str(mhz), "1965", "990.0", "Not Active", "Not Active", "Not Active", cap]  # noqa: E731
    samples = [(0.0, idle), (10.0, busy(1700, "Active")), (10.1, busy(1800, "Not Active")),
               (10.2, busy(1750, "Active")), (20.0, idle)]
    r = _sampler(samples).stop(10.0, 10.2)
    assert r["sm_mhz"] == 1750 and r["sm_max_mhz"] == 1965
    assert r["reasons"] == ["sw_power_cap"] and r["samples"] == 3


def test_clock_sampler_reports_throttling_and_missing_samples():
    hot = ["1200", "1965", "700.0", "Not Active", "Active", "Not Active", "Not Active"]
    r = _sampler([(5.0, hot)]).stop(5.0, 5.0)
    assert r["reasons"] == ["hw_thermal_slowdown"]
    # no sample inside the window: fall back to all samples
    assert _sampler([(1.0, hot)]).stop(5.0, 6.0)["sm_mhz"] == 1200
    assert _sampler([]).stop(0.0, 1.0)["reasons"] == ["no nvidia-smi samples"]


def test_recorded_traffic_matches_kernel_workload_and_source_hash():
    rows = [ln for ln in open(os.path.join(ROOT, "profiles", "dram_traffic.txt")) if ln.startswith("kernel=")]
    assert rows, "no traffic records"
    sha = bench.gemm_source_sha()
    for ln in rows:
        f = dict(kv.split("=", 1) for kv in ln.split())
        got, src = bench.recorded_traffic(f["kernel"], f["workload"])
        if f["source_sha"] == sha:
            assert got == float(f["dram_bytes_per_launch"]) and f["workload"] in src
            # a reduced-case record scales to the workloads it names
            for w in filter(None, f.get("scale_to", "").split(",")):
                alg = 2.0 * float(f["algorithmic_bytes"])
                scaled, src2 = bench.recorded_traffic(f["kernel"], w, alg)
                assert scaled == pytest.approx(2.0 * float(f["dram_bytes_per_launch"])) and "scaled" in src2
    assert bench.recorded_traffic("grouped_fp4_gemm_kernel<0>", "no-such-workload") == (None, None)


def test_source_hash_ignores_comments_but_not_code():
    src = "int a = 1;  // one\n/* a\n   block */\nint b = 2;\n\n// only a comment\n"
    assert bench._code_only(src) == "int a = 1;\nint b = 2;"
    assert bench._code_only(src.replace("// one", "// uno")) == bench._code_only(src)
    assert bench._code_only(src.replace("2;", "3;")) != bench._code_only(src)


def test_weak_scaling_value_counts_every_rank():
    # 16 tokens per rank, 4 ranks, 0.25 ms for the slowest rank's step
    assert bench.weak_scaling_value(16, 4, 0.25) == pytest.approx(16 * 4 / 0.25e-3)
