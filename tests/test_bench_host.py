"""Host-side parts of bench.py that need no GPU: the reference arm's JSON
line (the oracle timed on the host cores, bounded), the clock summary and the
peak denominators."""

import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


def test_reference_arm_line():
    d = _run("--impl", "reference", "--steps", "1", "--warmup", "3", "--workload", "c1")
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["warmup"] == 3  # K timed steps after W untimed ones
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == "c1_nvfp4_256x1024x1024"


def test_reference_arm_for_the_stack_is_unavailable():
    d = _run("--impl", "reference", "--workload", "c5")
    assert d["impl"] == "reference" and "unavailable" in d


def test_clock_summary_flags_throttling_and_counts_windows():
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s._h, s.max_mhz, s.period = object(), 1965, 0.0002
    # (host time, SM MHz, reason bits): sw_power_cap once, gpu_idle (not reported) once
    s.samples = [(0.0, 1800, 0x1), (1.0, 1900, 0x4), (2.0, 1965, 0), (3.0, 1500, 0)]
    s.windows = {}
    s.mark("headline", 0.5, 2.5)
    s.mark("other", 2.5, 3.5)
    out = s.summary("headline")
    assert out["sm_mhz"] == 1850.0 and out["samples"] == 4 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"]
    assert out["windows"]["headline"] == {"sm_mhz": 1932.5, "reasons": ["sw_power_cap"], "samples": 2,
                                          "sm_mhz_min": 1900}
    assert out["windows"]["other"]["samples"] == 1 and out["windows"]["other"]["reasons"] == []
    assert out["sm_mhz_headline"] == 1932.5 and out["samples_headline"] == 2
    s._h = None
    assert s.summary()["reasons"] == ["unavailable"]


def test_samples_are_taken_until_the_timed_region_ends():
    # the main thread samples while the last steps run (a fake event that
    # completes on its fourth query, a fake NVML)
    class Ev:
        n = 0

        def query(self):
            Ev.n += 1
            return Ev.n > 3

    class NV:
        NVML_CLOCK_SM = 0

        @staticmethod
        def nvmlDeviceGetClockInfo(h, which):
            return 1965

        @staticmethod
        def nvmlDeviceGetCurrentClocksEventReasons(h):
            return 0x4

    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s._h, s._nv, s.samples = object(), NV, []
    s.sample_until(Ev())
    assert len(s.samples) == 3 and all(m == 1965 and r == 0x4 for _, m, r in s.samples)
    s._h = None
    s.sample_until(Ev())  # no NVML: nothing, no error
    assert len(s.samples) == 3


def test_sustained_peak_needs_a_long_timed_region():
    # the denominator switches to the sustained figure only for a GEMM timed
    # inside a region of at least a second
    assert bench.SUSTAINED_MIN_MS >= 1000.0
    assert bench.NOMINAL_RATIO == {"nvfp4": 4.0, "mxfp8": 2.0, "bf16": 1.0}


def test_peaks_come_from_the_measured_file_or_the_fallback():
    p = bench._peaks()
    assert p["source"] in ("measured", "fallback")
    assert p["bf16"] > 0 and p["bf16_sustained"] > 0 and p["hbm"] > 0
    assert bench.whole_job_tflops(2, 10, 1e12, 1000.0) == 20.0


def test_c1_line_takes_the_nvfp4_path_it_names():
    # C1 (NVFP4 W4A4, 256 x 1024 x 1024) is below the selective rule's 1024:
    # the bench passes min_dim = 1 so that the step runs (and the line
    # reports) the NVFP4 path; mxq_linear_path is host logic on the weight
    # descriptor, so no device is needed
    import bench
    import workloads

    import fp8_gemm_diffusion_b200 as mxq

    name = workloads.CASE_NAMES["c1"]
    w = mxq.mxq_weight(format=mxq.NVFP4, flags=0, N=1024, K=1024)
    assert bench.default_min_dim(name, None) == 1
    assert mxq.linear_path(w, 256, bench.default_min_dim(name, None)) == mxq.NVFP4
    assert mxq.linear_path(w, 256, None) == mxq.BF16  # the library default keeps it in bf16
    assert bench.default_min_dim(workloads.CASE_NAMES["c3"], None) is None
    assert bench.default_min_dim(name, 4096) == 4096
