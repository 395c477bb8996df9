"""Benchmark of the microscaled linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c3|c2|c4|c1|c5|attn|bf16]
                    [--batch 1|4] [--impl mxq|reference] [--shape M,K,N --fmt nvfp4|mxfp8]

A step is one pass of the whole hot path over one batch of synthetic input:
for NVFP4, activation amax -> NVFP4 quantisation -> block-scaled GEMM with the
bias epilogue; for MXFP8, quantisation -> GEMM.  Weights are quantised once,
before timing (offline, as the method prescribes).  The default workload is
the NVFP4 MLP-up layer M=4608, K=3072, N=12288 (bias, 0.1 % outlier
channels).  The metric is TFLOP/s of the GEMM (2MNK per step) including the
activation quantisation.

Timing: W untimed warm-up steps; K timed steps bracketed by a barrier and
torch.cuda.synchronize(); CUDA events on the launching stream; max over
ranks.  The GEMM's own duration (the roofline's kernel) comes from an event
pair that mxq_linear records around its GEMM launch in every timed step.  Each step uses one of several rotating buffer sets whose total size
is well above the 126 MB L2, so no step starts with its inputs in L2.  Under
torchrun each rank runs an independent replica (weak scaling: no data-path
collective between replicas).

--workload c5 times a whole FLUX-shaped linear stack instead (about 300
layers per pass, mixed NVFP4 / bf16 by the selective rule; eager and replayed
from a CUDA graph) against the same stack in bf16 through cuBLAS; use a small
--steps there (one pass is ~17 ms at batch 1).  --workload attn times the
8-bit attention (24 heads x 4608 tokens x 128) against bf16 SDPA;
--workload bf16 times the dispatcher's bf16 branch against torch.addmm on
the stack's bf16 layers; --workload mlp4 times the NVFP4 MLP pair at
M = 16896 with the producer-fed amax (GELU epilogue + max|y|) and without.

--impl reference times the CPU oracle (the plain numpy restatement of the
method) on the host cores: W untimed and K timed steps, each a bounded sample
of the same workload (row chunks through amax, quantisation and the float64
GEMM), the budget per step sized so that the whole run takes a few minutes.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "block-scaled GEMM TFLOPS incl. act quant; % of dense FP4/FP8 peak"
UNIT = "TFLOP/s"
L2_BYTES = 126 * 1024 * 1024
# GPU spin ahead of each timed region (cycles; ~0.5 ms): the host gets ahead
SPIN_CYCLES = 1_000_000
# a GEMM timed inside a region at least this long is held to the sustained peak
SUSTAINED_MIN_MS = 1000.0
# Dense tensor peaks (TFLOP/s) for the roofline: the measured cuBLAS bf16
# figure of this machine pool times the nominal FP4:BF16 (4x) / FP8:BF16 (2x)
# ratio of B200; fallback numbers when no measurement file is present.
NOMINAL_RATIO = {"nvfp4": 4.0, "mxfp8": 2.0, "bf16": 1.0}


# DRAM bytes (read + write) of one launch of the roofline's kernel, from one
# ncu capture of the committed kernel (dram__bytes_read.sum +
# dram__bytes_write.sum); None where no capture of the current kernel exists.
GEMM_TRAFFIC_BYTES = {"c3_nvfp4_4608x3072x12288": 92199680, "c2_mxfp8_4608x3072x9216": 87975936,
                      "c4_nvfp4_16896x12288x3072": 222627840}


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(bf16=float(p["bf16_tflops"]), bf16_sustained=float(p["bf16_tflops_sustained"]),
                    hbm=float(p["hbm_gbs"]), source="measured")
    except Exception:
        return dict(bf16=1590.0, bf16_sustained=1400.0, hbm=6650.0, source="fallback")


# ---------------------------------------------------------------- clocks
def _nvml_id(local_rank: int):
    """NVML index (int) or UUID (str) of this rank's GPU."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if not vis:
        return local_rank
    entry = vis.split(",")[local_rank].strip()
    return int(entry) if entry.isdigit() else entry


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running.

    Every sample carries a host timestamp, so that a caller can count the
    samples that fell inside a given window (``mark``) as well as those of
    the whole measurement."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device, period_s: float = 0.0002):
        self.period = period_s
        self.samples = []  # (host time, SM MHz, reason bits)
        self.windows = {}
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = (pynvml.nvmlDeviceGetHandleByIndex(device) if isinstance(device, int)
                       else pynvml.nvmlDeviceGetHandleByUUID(device))
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._h = None

    def _sample(self):
        nv = self._nv
        self.samples.append((time.perf_counter(), nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM),
                             nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)))

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                break
            time.sleep(self.period)

    def start(self):
        if self._h is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def sample_until(self, event, max_s: float = 5.0):
        """Sample from the calling thread until `event` has completed: the
        timed region's last milliseconds, after the host has enqueued its
        work, while the sampler thread may still be waiting for the
        interpreter lock."""
        if self._h is None:
            return
        t0 = time.perf_counter()
        while not event.query() and time.perf_counter() - t0 < max_s:
            try:
                self._sample()
            except Exception:
                return

    def mark(self, name, t0, t1):
        """Record [t0, t1] (host perf_counter times) as a named window."""
        self.windows[name] = (t0, t1)

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()

    def _summ(self, samples):
        mhz = [m for _, m, _ in samples]
        bits = 0
        for _, _, r in samples:
            bits |= r
        names = [n for b, n in self.REASONS.items() if bits & b and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(mhz)) if mhz else None, "reasons": names,
                "samples": len(mhz), "sm_mhz_min": min(mhz) if mhz else None}

    def summary(self, window=None):
        """Median SM clock and the reasons seen, over all samples, with the
        counts inside each marked window (``window`` picks the headline one)."""
        if self._h is None or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        out = self._summ(self.samples)
        out["sm_max_mhz"] = self.max_mhz
        out["period_ms"] = self.period * 1e3
        out["windows"] = {}
        for name, (t0, t1) in self.windows.items():
            out["windows"][name] = self._summ([x for x in self.samples if t0 <= x[0] <= t1])
        if window in self.windows and out["windows"][window]["samples"]:
            w = out["windows"][window]
            out["sm_mhz_headline"] = w["sm_mhz"]
            out["samples_headline"] = w["samples"]
        return out


# ------------------------------------------------------- rank aggregation
def max_over_ranks(ms: float, device) -> float:
    """Max of a per-rank time over all ranks (identity without a process group)."""
    import torch.distributed as tdist
    if not (tdist.is_available() and tdist.is_initialized()) or tdist.get_world_size() == 1:
        return float(ms)
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world: int, steps: int, flops_per_step: float, max_ms: float) -> float:
    """Whole-job throughput: every replica did `steps` steps in at most max_ms."""
    return world * steps * flops_per_step / (max_ms * 1e-3) / 1e12


# ------------------------------------------------------------ the GPU arm
def default_min_dim(case_name: str, requested):
    """min_dim passed to mxq_linear: the caller's, else 1 for C1 (the NVFP4 W4A4
    single-GEMM configuration, 256 x 1024 x 1024, which the selective rule
    would otherwise keep in bf16), else the library's default (None)."""
    if requested is not None:
        return requested
    return 1 if case_name.startswith("c1") else None


def run_gpu(args, rank, world, local_rank):
    import fp8_gemm_diffusion_b200 as mxq

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if args.shape:
        Ms, Ks, Ns = (int(v) for v in args.shape.split(","))
        case = workloads.random_case(Ms, Ks, Ns, args.fmt, seed=0)
    else:
        case = workloads.make_case(args.workload)
    fmt = case.fmt
    M, K, N = case.M, case.K, case.N
    flops = 2.0 * M * N * K
    stream = torch.cuda.current_stream(dev)

    # one prepared weight, then per-set copies of everything a step touches
    W = case.W.to(dev)
    bias = case.bias.to(dev) if case.bias is not None else None
    # NVFP4 without a per-tensor scale (g = 1, no amax pass) on request
    unit_g = fmt == "nvfp4" and args.no_tensor_scale
    base_w = mxq.Weight(W, bias, fmt=fmt, tensor_scale=not unit_g)
    ws_bytes = mxq.linear_workspace_bytes(M, K, fmt)
    per_set = M * K * 2 + mxq.weight_storage_bytes(N, K, fmt) + M * N * 2 + ws_bytes
    nsets = max(2, int(np.ceil(3 * L2_BYTES / per_set)))
    A0 = case.A.to(dev)
    sets = []
    for _ in range(nsets):
        storage = base_w.storage.clone()
        h = mxq.mxq_weight.from_buffer_copy(base_w.handle)
        off = storage.data_ptr() - base_w.storage.data_ptr()
        h.codes += off
        h.sf += off
        if h.g_dev:
            h.g_dev += off
            h.amax_dev += off
        sets.append(dict(x=A0.clone(), storage=storage, w=h,
                         y=torch.empty(M, N, dtype=torch.bfloat16, device=dev),
                         ws=torch.empty(ws_bytes, dtype=torch.uint8, device=dev)))
    # the activation quantised once through the public calls, for the GEMM-only timing
    qa_codes = torch.empty(mxq.codes_bytes(M, K, fmt), dtype=torch.uint8, device=dev)
    qa_sf = torch.empty(mxq.sf_bytes(M, K, fmt), dtype=torch.uint8, device=dev)
    qa_amax = torch.empty(1, dtype=torch.float32, device=dev)
    qa_g = torch.empty(1, dtype=torch.float32, device=dev)

    def quantize_public(x):
        if fmt == "nvfp4":
            mxq.amax(x, qa_amax, stream=stream)
            mxq.quantize_nvfp4(x, qa_amax, qa_codes, qa_sf, qa_g, stream=stream)
        else:
            mxq.quantize_mxfp8(x, qa_codes, qa_sf, stream=stream)

    quantize_public(A0)
    torch.cuda.synchronize()

    # The path the dispatcher takes for this layer.  C1 is the NVFP4 W4A4
    # single-GEMM configuration: its 256 x 1024 x 1024 shape is below the
    # selective rule's 1024 threshold, so it is run with min_dim = 1 to time
    # the NVFP4 path it names (the line reports the path actually taken).
    min_dim = default_min_dim(case.name, args.min_dim)
    path = mxq.linear_path(base_w.handle, M, min_dim)
    run_fmt = {mxq.NVFP4: "nvfp4", mxq.MXFP8: "mxfp8", mxq.BF16: "bf16"}[path]

    def step(i, gemm_events=None):
        st = sets[i % nsets]
        mxq.linear(st["w"], st["x"], M, st["y"], st["ws"], ws_bytes, stream=stream,
                   gemm_events=gemm_events, min_dim=min_dim)

    def gemm_only(i):
        st = sets[i % nsets]
        h = st["w"]
        mxq.gemm_blockscaled(fmt, M, N, K, qa_codes, qa_sf, qa_g if fmt == "nvfp4" else None,
                             h.codes, h.sf, h.g_dev if fmt == "nvfp4" else None, bias, st["y"],
                             stream=stream)

    # kernels one mxq_linear call launches here (the library's own dispatch decision)
    launches_per_step = mxq.linear_kernel_count(base_w.handle, M, min_dim)
    assert launches_per_step > 0, launches_per_step
    dist = world > 1
    if dist:
        import torch.distributed as tdist
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if mxq.get_device_error() != mxq.OK:
        raise RuntimeError("device-side timeout during warm-up")

    # one event pair per timed step, recorded by mxq_linear around its GEMM launch
    # (created here: torch creates an event's handle on its first record)
    gemm_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(args.steps)]
    for a, b in gemm_evs:
        a.record(stream)
        b.record(stream)
    torch.cuda.synchronize()
    sampler = ClockSampler(_nvml_id(local_rank))
    sampler.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)

    def timed_pass(name, n, fn):
        """n calls of fn(i) between two events; max over ranks of the span.
        A short spin kernel ahead of the start event lets the host enqueue the
        first steps before the GPU reaches them, so the span holds GPU work
        only (no launch gap at its start)."""
        if dist:
            tdist.barrier()
        torch.cuda.synchronize()
        torch.cuda._sleep(SPIN_CYCLES)
        t_start.record(stream)
        h0 = time.perf_counter()
        for i in range(n):
            fn(i)
        t_end.record(stream)
        sampler.sample_until(t_end)
        torch.cuda.synchronize()
        sampler.mark(name, h0, time.perf_counter())
        if dist:
            tdist.barrier()
        return max_over_ranks(t_start.elapsed_time(t_end), dev)

    total_ms = timed_pass("headline", args.steps, lambda i: step(args.warmup + i))
    if mxq.get_device_error() != mxq.OK:
        raise RuntimeError("device-side timeout during the timed steps")

    # second pass of the same K steps with an event pair around every GEMM
    # launch: the GEMM's average duration inside the steps (the roofline's
    # kernel).  An event recorded between two kernels costs the next one its
    # programmatic early launch, so the headline value comes from the first pass.
    total_ev_ms = timed_pass("gemm_events", args.steps, lambda i: step(args.warmup + i, gemm_evs[i]))
    gemm_ms = float(np.mean([a.elapsed_time(b) for a, b in gemm_evs]))
    if mxq.get_device_error() != mxq.OK:
        raise RuntimeError("device-side timeout during the timed steps")

    # the same step with one buffer set only (inputs stay in L2 between steps):
    # the hot number beside the L2-cold headline
    hot_steps = max(10, min(args.steps, 500))
    hot_ms = timed_pass("hot", hot_steps, lambda i: step(0)) / hot_steps
    sampler.stop()

    # for comparison: the GEMM launched alone, back to back, same stream
    reps = max(10, min(args.steps, 50))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
    for i in range(reps):
        evs[i][0].record(stream)
        gemm_only(i)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    gemm_alone_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    for i in range(reps):
        evs[i][0].record(stream)
        quantize_public(sets[i % nsets]["x"])
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    quant_pub_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))

    # bf16 tensor-core baseline in the same run: cuBLAS (torch.addmm) on the
    # same shape, bias and rotating buffers, timed the same way
    bf16_ms = bf16_baseline_ms(sets, W, bias, M, N, stream, args.warmup, min(args.steps, 500), dev, dist)

    # end to end through the public call with host buffers
    e2e = run_e2e(mxq, case, base_w, dev, stream, args, dist)

    peaks = _peaks()
    # The denominator follows the timed region's length: the burst figure
    # (cuBLAS timed alone) unless the GEMM ran inside a region of at least a
    # second, long enough for the power cap to settle the clock (the sustained
    # figure).  The other one is reported beside it.
    sustained = total_ev_ms >= SUSTAINED_MIN_MS
    peak_burst = peaks["bf16"] * NOMINAL_RATIO[run_fmt]
    peak_sus = peaks["bf16_sustained"] * NOMINAL_RATIO[run_fmt]
    peak = peak_sus if sustained else peak_burst
    achieved = flops / (gemm_ms * 1e-3) / 1e12
    clocks = sampler.summary("headline")
    gemm_mhz = (clocks.get("windows", {}).get("gemm_events", {}) or {}).get("sm_mhz")
    value = whole_job_tflops(world, args.steps, flops, total_ms)
    bf16_tflops = whole_job_tflops(world, 1, flops, bf16_ms)
    step_ms = total_ms / args.steps
    qbytes = M * K * 2 + mxq.codes_bytes(M, K, run_fmt) + mxq.sf_bytes(M, K, run_fmt)
    nominal = {"nvfp4": 9000.0, "mxfp8": 4500.0, "bf16": 2250.0}[run_fmt]
    step_text = {"nvfp4": "mxq_linear: activation amax + NVFP4 quantisation + block-scaled GEMM "
                          "(weights pre-quantised)",
                 "mxfp8": "mxq_linear: MXFP8 activation quantisation + block-scaled GEMM "
                          "(weights pre-quantised)",
                 "bf16": "mxq_linear: bf16 GEMM (selective rule)"}[run_fmt]
    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": {"nvfp4": "e2m1+e4m3 (nvfp4), fp32 accumulate, bf16 out",
                  "mxfp8": "e4m3+e8m0 (mxfp8), fp32 accumulate, bf16 out",
                  "bf16": "bf16, fp32 accumulate, bf16 out"}[run_fmt],
        "data": "synthetic (seeded, FLUX-shaped; random-init weights)",
        "config": {
            "workload": case.name, "format": fmt, "path": run_fmt,
            "min_dim": min_dim if min_dim is not None else 1024, "M": M, "K": K, "N": N,
            "bias": case.bias is not None, "per_tensor_scale": not unit_g,
            "parallelism": f"replicas x{world}",
            "step": step_text,
            "l2": f"rotating {nsets} buffer sets ({nsets * per_set / 2**20:.0f} MiB > 126 MiB L2)",
        },
        "fraction_of_dense_peak": {"nominal": round(value / nominal, 4), "nominal_peak_tflops": nominal},
        "kernels_ms": {
            "gemm": round(gemm_ms, 5),
            "quantize_in_step": round(step_ms - gemm_ms, 5),
            "step_with_gemm_events": round(total_ev_ms / args.steps, 5),
            "gemm_alone": round(gemm_alone_ms, 5),
            "quantize_public_calls": round(quant_pub_ms, 5),
        },
        "quantize_gbs": round(qbytes / (max(step_ms - gemm_ms, 1e-6) * 1e-3) / 1e9, 1),
        "quantize_note": "algorithmic bytes over quantize_in_step = the step (launches overlapping through "
                         "programmatic dependent launch) minus the GEMM timed with events around it (which "
                         "costs it that overlap): the quantiser's share of the step, not its standalone "
                         "duration (quantize_public_calls times the public calls alone, launch gaps included)",
        "hot": {"value": round(whole_job_tflops(world, 1, flops, hot_ms), 2), "unit": UNIT,
                "ms_per_step": round(hot_ms, 5), "steps": hot_steps,
                "l2": "one buffer set reused every step (inputs L2-resident)"},
        "roofline": {
            "kernel": f"gemm_pair_kernel<{run_fmt}>" if M > 128 else f"gemm_kernel<{run_fmt}>",
            "bound": "tensor",
            "achieved": round(achieved, 2),
            "peak": round(peak, 1),
            "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4),
            "peak_kind": "sustained" if sustained else "burst",
            "peak_source": f"{peaks['source']} bf16 {'sustained' if sustained else 'burst'} "
                           f"{peaks['bf16_sustained'] if sustained else peaks['bf16']} TFLOP/s x "
                           f"{NOMINAL_RATIO[run_fmt]:g} (nominal {run_fmt}:bf16 dense ratio); "
                           f"{'sustained' if sustained else 'burst'} because the GEMM's timed region "
                           f"was {total_ev_ms:.1f} ms ({'>=' if sustained else '<'} "
                           f"{SUSTAINED_MIN_MS:.0f} ms); the GEMM is timed by events around its "
                           f"launch inside the timed steps",
            "peak_other": round(peak_burst if sustained else peak_sus, 1),
            "frac_of_other": round(achieved / (peak_burst if sustained else peak_sus), 4),
            "frac_of_nominal": round(achieved / nominal, 4),
            "gemm_cycles_per_launch": round(gemm_ms * 1e-3 * gemm_mhz * 1e6) if gemm_mhz else None,
            "gemm_cycles_note": "in-step GEMM time x median SM clock sampled during that pass",
            "traffic": GEMM_TRAFFIC_BYTES.get(case.name),
            "traffic_unit": "bytes per launch (ncu dram read + write)",
        },
        "bf16_baseline": {
            "impl": "torch.addmm bf16 (cuBLAS), same shape, bias and buffers",
            "value": round(bf16_tflops, 2), "unit": UNIT,
            "ms_per_step": round(bf16_ms, 5),
            "speedup_of_value": round(value / bf16_tflops, 3),
            "fraction_of_dense_peak": {"nominal": round(bf16_tflops / 2250.0, 4),
                                       "nominal_peak_tflops": 2250.0,
                                       "measured_burst": round(bf16_tflops / peaks["bf16"], 4)},
        },
        "clocks": clocks,
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
    }
    return result


def bf16_baseline_ms(sets, W, bias, M, N, stream, warmup, steps, dev, dist):
    """Average step time of y = x W^T + bias in bf16 through cuBLAS (torch.addmm),
    over the bench's rotating activation / output buffers."""
    Wt = W.t()
    b = bias if bias is not None else torch.zeros(N, dtype=torch.bfloat16, device=W.device)
    with torch.cuda.stream(stream):
        for i in range(warmup):
            st = sets[i % len(sets)]
            torch.addmm(b, st["x"], Wt, out=st["y"])
        torch.cuda.synchronize()
        if dist:
            import torch.distributed as tdist
            tdist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(steps):
            st = sets[i % len(sets)]
            torch.addmm(b, st["x"], Wt, out=st["y"])
        e1.record(stream)
        torch.cuda.synchronize()
    return max_over_ranks(e0.elapsed_time(e1), dev) / steps


def run_e2e(mxq, case, base_w, dev, stream, args, dist):
    """Same metric through mxq_linear with pinned host input and output:
    each step copies A host->device, runs the layer, copies Y device->host."""
    M, K, N = case.M, case.K, case.N
    fmt = case.fmt
    x_host = case.A.pin_memory()
    y_host = torch.empty(M, N, dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    y_dev = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    ws_bytes = mxq.linear_workspace_bytes(M, K, fmt)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    steps = max(3, min(args.steps, 20))

    def one():
        x_dev.copy_(x_host, non_blocking=True)
        mxq.linear(base_w.handle, x_dev, M, y_dev, ws, ws_bytes, stream=stream)
        y_host.copy_(y_dev, non_blocking=True)

    for _ in range(2):
        one()
    torch.cuda.synchronize()
    if dist:
        import torch.distributed as tdist
        tdist.barrier()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        one()
    b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b), dev)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    flops = 2.0 * M * N * K
    return {"value": round(whole_job_tflops(world, steps, flops, ms), 3), "unit": UNIT,
            "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2, "steps": steps}


# ------------------------------------------------- the FLUX linear stack
def run_stack(args, rank, world, local_rank):
    """One step = one forward pass over every linear layer of the FLUX-shaped
    DiT stack (19 double-stream + 38 single-stream blocks) in forward order,
    each through mxq_linear with the selective rule (bf16 below the 1024
    threshold, NVFP4 otherwise), quantisation of every NVFP4 layer's
    activation included.  Seeded random weights (N(0, 0.02), bias N(0, 0.02))
    and one N(0, 1) activation buffer per distinct (M, K); the 6+ GB of
    weights stream from HBM in every pass.  Timed eagerly and, when the pass
    can be captured, replayed from one CUDA graph; the same stack in bf16
    through cuBLAS (torch.addmm) is timed the same way."""
    import fp8_gemm_diffusion_b200 as mxq

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    layers = workloads.flux_linear_stack(batch=args.batch)
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    acts, outs, prepared = {}, {}, []
    flops = flops_q = 0.0
    ws_bytes = 256
    launches = 0
    for l in layers:
        M, K, N = l["M"], l["K"], l["N"]
        if (M, K) not in acts:
            acts[(M, K)] = torch.randn(M, K, generator=g, device=dev).to(torch.bfloat16)
        if (M, N) not in outs:
            outs[(M, N)] = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        W = (torch.randn(N, K, generator=g, device=dev) * 0.02).to(torch.bfloat16)
        b = (torch.randn(N, generator=g, device=dev) * 0.02).to(torch.bfloat16)
        w = mxq.Weight(W, b, fmt="nvfp4")
        path = mxq.linear_path(w.handle, M)
        if path != mxq.BF16:
            ws_bytes = max(ws_bytes, mxq.linear_workspace_bytes(M, K, path))
            flops_q += 2.0 * M * N * K
        flops += 2.0 * M * N * K
        launches += mxq.linear_kernel_count(w.handle, M)
        prepared.append((w, acts[(M, K)], M, outs[(M, N)], W, b))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()

    def one_pass():
        s = torch.cuda.current_stream(dev)
        for w, x, M, y, _, _ in prepared:
            mxq.linear(w.handle, x, M, y, ws, ws_bytes, stream=s)

    def bf16_pass():
        for _, x, _, y, W, b in prepared:
            torch.addmm(b, x, W.t(), out=y)

    def timed(fn, steps):
        torch.cuda.synchronize()
        if world > 1:
            import torch.distributed as tdist
            tdist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(e0.elapsed_time(e1), dev)

    for _ in range(args.warmup):
        one_pass()
    torch.cuda.synchronize()
    if mxq.get_device_error() != mxq.OK:
        raise RuntimeError("device-side timeout during warm-up")
    sampler = ClockSampler(_nvml_id(local_rank))
    sampler.start()
    eager_ms = timed(one_pass, args.steps)
    sampler.stop()
    if mxq.get_device_error() != mxq.OK:
        raise RuntimeError("device-side timeout during the timed passes")

    graph_ms, graph_note = None, None
    try:
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            one_pass()  # warm the side stream
        stream.wait_stream(side)
        torch.cuda.synchronize()
        with torch.cuda.graph(graph):
            one_pass()
        for _ in range(2):
            graph.replay()
        graph_ms = timed(graph.replay, args.steps)
        if mxq.get_device_error() != mxq.OK:
            raise RuntimeError("device-side timeout during the graph replays")
        del graph
    except Exception as e:  # capture unsupported: report it, keep the eager number
        graph_note = f"not captured: {type(e).__name__}: {str(e).splitlines()[0][:160]}"
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        bf16_pass()
    bf16_ms = timed(bf16_pass, max(1, min(args.steps, 20))) / max(1, min(args.steps, 20))
    best_ms = min(eager_ms, graph_ms) if graph_ms is not None else eager_ms
    pass_ms = best_ms / args.steps
    value = whole_job_tflops(world, 1, flops, pass_ms)
    peaks = _peaks()
    sustained = best_ms >= SUSTAINED_MIN_MS
    peak = (peaks["bf16_sustained"] if sustained else peaks["bf16"]) * NOMINAL_RATIO["nvfp4"]
    return {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(pass_ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "mixed: e2m1+e4m3 (nvfp4) where quantised, bf16 elsewhere; fp32 accumulate, bf16 out",
        "data": "synthetic (seeded, FLUX-shaped stack; random-init weights)",
        "config": {
            "workload": f"c5_flux_linear_stack_b{args.batch}", "layers": len(layers),
            "quantised_flop_fraction": round(flops_q / flops, 5),
            "parallelism": f"replicas x{world}",
            "step": "one forward pass over the stack through mxq_linear (selective rule)",
            "timed_as": "cuda graph replay" if graph_ms is not None and graph_ms <= eager_ms else "eager",
            "l2": "weights (> 6 GB) stream from HBM every pass; activation buffers are reused",
        },
        "fraction_of_dense_peak": {"nominal": round(value / 9000.0, 4), "nominal_peak_tflops": 9000.0},
        "stack_ms": {"eager": round(eager_ms / args.steps, 4),
                     "graph": round(graph_ms / args.steps, 4) if graph_ms is not None else None,
                     "graph_note": graph_note},
        "roofline": {"kernel": "whole stack (mixed nvfp4 / bf16 GEMMs)", "bound": "tensor",
                     "achieved": round(value, 2), "peak": round(peak, 1), "unit": "TFLOP/s",
                     "frac": round(value / peak, 4), "traffic": None,
                     "peak_kind": "sustained" if sustained else "burst",
                     "peak_source": f"{peaks['source']} bf16 {'sustained' if sustained else 'burst'} x 4 "
                                    f"(nvfp4 dense ratio); timed region {best_ms:.0f} ms"},
        "bf16_baseline": {"impl": "torch.addmm bf16 (cuBLAS), the same stack, weights and buffers",
                          "value": round(whole_job_tflops(world, 1, flops, bf16_ms), 2), "unit": UNIT,
                          "ms_per_step": round(bf16_ms, 4),
                          "speedup_of_value": round(bf16_ms / pass_ms, 3)},
        "clocks": sampler.summary(),
        "e2e": None,
        "gpu_launches": launches * args.steps,
        "cpu_baseline": None,
    }


def run_bf16_branch(args, rank, world, local_rank):
    """The dispatcher's bf16 branch against cuBLAS.  Every distinct layer
    shape of the FLUX-shaped stack that the selective rule keeps in bf16
    (batch 1: the modulation layers at M = 1 and the text stream's layers at
    M = 512; batch 4: the modulation layers at M = 4) runs through
    mxq_linear (the library's own tcgen05 bf16 GEMM) and through torch.addmm
    on the same bf16 weights, bias and buffers.  Weight sets rotate so that
    more than 2 x L2 of weights stream between two uses of one set.  The
    line's value is the stack's bf16-layer flops over the summed per-layer
    time of the library, each shape weighted by its count in the stack."""
    import fp8_gemm_diffusion_b200 as mxq

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    counts = {}
    for l in workloads.flux_linear_stack(batch=args.batch):
        key = (l["M"], l["K"], l["N"])
        counts[key] = counts.get(key, 0) + 1
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    rows, launches = [], 0
    tot_flops = tot_mxq = tot_ref = 0.0
    probe = None
    for (M, K, N), cnt in counts.items():
        W0 = (torch.randn(N, K, generator=g, device=dev) * 0.02).to(torch.bfloat16)
        b0 = (torch.randn(N, generator=g, device=dev) * 0.02).to(torch.bfloat16)
        w0 = mxq.Weight(W0, b0, fmt="nvfp4")
        if mxq.linear_path(w0.handle, M) != mxq.BF16:
            continue
        nsets = max(2, -(-(256 << 20) // (N * K * 2)))
        sets = [(W0, b0, w0)] + [
            ((W := (torch.randn(N, K, generator=g, device=dev) * 0.02).to(torch.bfloat16)),
             (b := (torch.randn(N, generator=g, device=dev) * 0.02).to(torch.bfloat16)),
             mxq.Weight(W, b, fmt="nvfp4")) for _ in range(nsets - 1)]
        x = torch.randn(M, K, generator=g, device=dev).to(torch.bfloat16)
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        y_ref = torch.empty_like(y)
        ws_bytes = max(256, mxq.linear_workspace_bytes(M, K, mxq.BF16))
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)

        def ours(i, sets=sets, x=x, y=y, ws=ws, ws_bytes=ws_bytes, M=M):
            mxq.linear(sets[i % len(sets)][2].handle, x, M, y, ws, ws_bytes, stream=stream)

        def cublas(i, sets=sets, x=x, y_ref=y_ref):
            W, b, _ = sets[i % len(sets)]
            torch.addmm(b, x, W.t(), out=y_ref)

        def timed(fn, n):
            for i in range(args.warmup):
                fn(i)
            torch.cuda.synchronize()
            torch.cuda._sleep(SPIN_CYCLES)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for i in range(n):
                fn(i)
            e1.record(stream)
            torch.cuda.synchronize()
            return max_over_ranks(e0.elapsed_time(e1), dev) / n

        n = max(args.steps, 3 * nsets)
        ms_ours = timed(ours, n)
        ms_ref = timed(cublas, n)
        launches += n
        if mxq.get_device_error() != mxq.OK:
            raise RuntimeError("device-side timeout in the bf16 branch")
        ours(0)
        cublas(0)
        torch.cuda.synchronize()
        diff = (y.float() - y_ref.float()).abs().max().item()
        flops = 2.0 * M * N * K
        tot_flops += cnt * flops
        tot_mxq += cnt * ms_ours
        tot_ref += cnt * ms_ref
        rows.append({"M": M, "K": K, "N": N, "count_in_stack": cnt, "us_mxq": round(ms_ours * 1e3, 2),
                     "us_addmm": round(ms_ref * 1e3, 2), "addmm_over_mxq": round(ms_ref / ms_ours, 3),
                     "tflops_mxq": round(flops / (ms_ours * 1e-3) / 1e12, 1),
                     "weight_gbs_mxq": round(N * K * 2 / (ms_ours * 1e-3) / 1e9, 1),
                     "max_abs_diff_vs_addmm": diff})
    value = tot_flops / (tot_mxq * 1e-3) / 1e12
    peaks = _peaks()
    return {
        "metric": "bf16-branch GEMM TFLOPS over the FLUX stack's bf16 layers (stack-weighted)",
        "value": round(value, 2),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(tot_mxq, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 operands, fp32 accumulate, bf16 out",
        "data": "synthetic (seeded FLUX-shaped layers; random-init weights)",
        "config": {"workload": f"c5_bf16_layers_b{args.batch}", "parallelism": f"replicas x{world}",
                   "step": "each bf16-path layer of the stack once, through mxq_linear",
                   "l2": "rotating weight sets, > 256 MiB of weights between two uses of a set"},
        "per_shape": rows,
        "bf16_baseline": {"impl": "torch.addmm bf16 (cuBLAS), same weights and buffers",
                          "value": round(tot_flops / (tot_ref * 1e-3) / 1e12, 2), "unit": UNIT,
                          "ms_per_step": round(tot_ref, 5), "speedup_of_value": round(tot_ref / tot_mxq, 3)},
        "roofline": {"kernel": "gemm_kernel<BF16> / gemm_pair_kernel<BF16>", "bound": "hbm",
                     "note": "the M = 1 and M = 512 layers stream their weights; see per_shape weight_gbs_mxq",
                     "peak": peaks["hbm"], "unit": "GB/s", "achieved": None, "frac": None, "traffic": None},
        "e2e": None,
        "gpu_launches": launches,
        "cpu_baseline": None,
    }


def run_mlp(args, rank, world, local_rank):
    """One step = the NVFP4 MLP pair of a single-stream block at 2048 x 2048
    (M = 16896 tokens): mlp_up 3072 -> 12288 whose epilogue applies GELU, then
    mlp_down 12288 -> 3072 (the C4 layer) on that output, both through
    mxq_linear with their activation quantisation.  Timed two ways on the same
    buffers: producer-fed (mlp_up's epilogue also folds max |y| of its bf16
    output into one device word, and mlp_down's quantiser takes it instead of
    its own amax pass: one read of the 415 MB activation) and unfused (mlp_down
    takes its own amax: two reads).  The GEMMs' own durations come from event
    pairs mxq_linear records around them; the rest of the step is the two
    activation quantisations.  Seeded inputs: x ~ N(0, 1), weights ~ N(0,
    0.02) / N(0, 0.01), biases ~ N(0, 0.02)."""
    import fp8_gemm_diffusion_b200 as mxq

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    M, H, F = 16896, 3072, 12288
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    x = torch.randn(M, H, generator=g, device=dev).to(torch.bfloat16)
    W1 = (torch.randn(F, H, generator=g, device=dev) * 0.02).to(torch.bfloat16)
    b1 = (torch.randn(F, generator=g, device=dev) * 0.02).to(torch.bfloat16)
    W2 = (torch.randn(H, F, generator=g, device=dev) * 0.01).to(torch.bfloat16)
    b2 = (torch.randn(H, generator=g, device=dev) * 0.02).to(torch.bfloat16)
    w1 = mxq.Weight(W1, b1, fmt="nvfp4")
    w2 = mxq.Weight(W2, b2, fmt="nvfp4")
    del W1, W2
    h = torch.empty(M, F, dtype=torch.bfloat16, device=dev)
    y = torch.empty(M, H, dtype=torch.bfloat16, device=dev)
    ws1_bytes = mxq.linear_workspace_bytes(M, H, mxq.NVFP4)
    ws2_bytes = mxq.linear_workspace_bytes(M, F, mxq.NVFP4)
    ws1 = torch.empty(ws1_bytes, dtype=torch.uint8, device=dev)
    ws2 = torch.empty(ws2_bytes, dtype=torch.uint8, device=dev)
    h_amax = torch.zeros(1, dtype=torch.float32, device=dev)
    flops = 2.0 * M * H * F * 2
    launches = {True: mxq.linear_kernel_count(w1.handle, M) + mxq.linear_kernel_count(w2.handle, M, x_amax=h_amax),
                False: mxq.linear_kernel_count(w1.handle, M) + mxq.linear_kernel_count(w2.handle, M)}

    def step(fused, ev=None):
        e1 = ev[0] if ev else None
        e2 = ev[1] if ev else None
        mxq.linear(w1.handle, x, M, h, ws1, ws1_bytes, stream=stream, gemm_events=e1,
                   activation=mxq.ACT_GELU, y_amax=h_amax if fused else None)
        mxq.linear(w2.handle, h, M, y, ws2, ws2_bytes, stream=stream, gemm_events=e2,
                   x_amax=h_amax if fused else None)

    def timed(fn, n):
        if world > 1:
            import torch.distributed as tdist
            tdist.barrier()
        torch.cuda.synchronize()
        torch.cuda._sleep(SPIN_CYCLES)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(n):
            fn(i)
        e1.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(e0.elapsed_time(e1), dev)

    res = {}
    sampler = ClockSampler(_nvml_id(local_rank))
    sampler.start()
    for fused in (True, False):
        for _ in range(args.warmup):
            step(fused)
        torch.cuda.synchronize()
        if mxq.get_device_error() != mxq.OK:
            raise RuntimeError("device-side timeout during warm-up")
        t0 = time.perf_counter()
        ms = timed(lambda i: step(fused), args.steps) / args.steps
        sampler.mark("fused" if fused else "unfused", t0, time.perf_counter())
        evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(2)]
               for _ in range(args.steps)]
        for ev in evs:
            for a, b in ev:
                a.record(stream)
                b.record(stream)
        torch.cuda.synchronize()
        timed(lambda i: step(fused, evs[i]), args.steps)
        g1 = float(np.mean([ev[0][0].elapsed_time(ev[0][1]) for ev in evs]))
        g2 = float(np.mean([ev[1][0].elapsed_time(ev[1][1]) for ev in evs]))
        if mxq.get_device_error() != mxq.OK:
            raise RuntimeError("device-side timeout in the timed steps")
        res[fused] = dict(ms=ms, gemm_up_ms=g1, gemm_down_ms=g2)
    sampler.stop()
    fz, un = res[True], res[False]
    value = whole_job_tflops(world, 1, flops, fz["ms"])
    peaks = _peaks()
    peak = peaks["bf16"] * NOMINAL_RATIO["nvfp4"]

    def quant_share(r):
        q = max(0.0, r["ms"] - r["gemm_up_ms"] - r["gemm_down_ms"])
        return round(q * 1e3, 2), round(q / r["ms"], 4)

    return {
        "metric": "NVFP4 MLP-pair TFLOPS incl. activation quantisation (2 x 2MKN per step)",
        "value": round(value, 2),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(fz["ms"], 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 + e4m3 block scales + fp32 tensor scale); fp32 accumulate; bf16 out",
        "data": "synthetic (seeded; random-init weights)",
        "config": {"workload": "mlp_pair_16896x3072x12288_gelu", "M": M, "hidden": H, "mlp": F,
                   "parallelism": f"replicas x{world}",
                   "step": "mlp_up (GELU epilogue, max|y| folded into one word) -> mlp_down quantised with "
                           "that amax (one pass over its 415 MB input) -> GEMM",
                   "l2": "every buffer of a step (> 1 GB) is larger than L2"},
        "producer_fed": {"ms_per_step": round(fz["ms"], 5), "gemm_up_us": round(fz["gemm_up_ms"] * 1e3, 2),
                         "gemm_down_us": round(fz["gemm_down_ms"] * 1e3, 2),
                         "quantisation_us": quant_share(fz)[0], "quantisation_share": quant_share(fz)[1]},
        "unfused": {"ms_per_step": round(un["ms"], 5), "value": round(whole_job_tflops(world, 1, flops, un["ms"]), 2),
                    "gemm_up_us": round(un["gemm_up_ms"] * 1e3, 2), "gemm_down_us": round(un["gemm_down_ms"] * 1e3, 2),
                    "quantisation_us": quant_share(un)[0], "quantisation_share": quant_share(un)[1]},
        "speedup_of_fusion": round(un["ms"] / fz["ms"], 4),
        "roofline": {"kernel": "gemm_pair_kernel<NVFP4> x 2 + quantisers", "bound": "tensor",
                     "achieved": round(value, 2), "peak": round(peak, 1), "unit": "TFLOP/s",
                     "frac": round(value / peak, 4), "peak_kind": "burst",
                     "peak_source": f"{peaks['source']} bf16 burst x 4 (nvfp4 dense ratio); whole step",
                     "traffic": None},
        "clocks": sampler.summary("fused"),
        "e2e": None,
        "gpu_launches": launches[True] * args.steps,
        "cpu_baseline": None,
    }


# ------------------------------------------------------------- attention
def run_attention(args, rank, world, local_rank):
    """One step = one FLUX-shaped attention (24 heads x 4608 tokens x 128)
    through mxq_attention_mxfp8: per-token MXFP8 of Q and K, MXFP8 of V^T,
    then the attention kernel (one pass over the keys).  The metric counts
    the attention's two products, 4 * heads * tokens^2 * d per step, which
    is also what the tensor cores run.  Baseline: PyTorch's
    scaled_dot_product_attention in bf16 on the same tensors."""
    import torch.nn.functional as Fn

    import fp8_gemm_diffusion_b200 as mxq

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    H, T, d = 24, 4608, 128
    Q, K, V = (t.to(dev) for t in workloads.flux_attention(H, T, d))
    nsets = 4  # 4 x 85 MB of inputs rotate: no step starts with its inputs in L2
    sets = [(Q.clone(), K.clone(), V.clone(), torch.empty_like(Q)) for _ in range(nsets)]
    nbytes = mxq.attention_workspace_bytes(H, T, d)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    flops = 4.0 * H * T * T * d
    mma_flops = flops

    def step(i):
        q, k, v, o = sets[i % nsets]
        mxq.attention_mxfp8(q, k, v, H, T, o, ws, nbytes, stream=stream)

    def timed(fn, n):
        if world > 1:
            import torch.distributed as tdist
            tdist.barrier()
        torch.cuda.synchronize()
        torch.cuda._sleep(SPIN_CYCLES)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(n):
            fn(i)
        e1.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(e0.elapsed_time(e1), dev)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if mxq.get_device_error() != mxq.OK:
        raise RuntimeError("device-side timeout during warm-up")
    sampler = ClockSampler(_nvml_id(local_rank))
    sampler.start()
    t0 = time.perf_counter()
    total_ms = timed(step, args.steps)
    sampler.mark("headline", t0, time.perf_counter())
    # the attention kernel alone (the quantisers' share is the rest of the step)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(10)]
    for i, (a, b) in enumerate(evs):
        q, k, v, o = sets[i % nsets]
        a.record(stream)
        step(i)
        b.record(stream)
    torch.cuda.synchronize()
    sampler.stop()
    call_ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    if mxq.get_device_error() != mxq.OK:
        raise RuntimeError("device-side timeout during the timed steps")

    def sdpa(i):
        q, k, v, o = sets[i % nsets]
        o.copy_(Fn.scaled_dot_product_attention(q.unsqueeze(0), k.unsqueeze(0), v.unsqueeze(0))[0])

    for i in range(args.warmup):
        sdpa(i)
    bf16_ms = timed(sdpa, max(1, min(args.steps, 50))) / max(1, min(args.steps, 50))
    step_ms = total_ms / args.steps
    value = whole_job_tflops(world, 1, flops, step_ms)
    peaks = _peaks()
    peak = peaks["bf16"] * NOMINAL_RATIO["mxfp8"]
    return {
        "metric": "8-bit attention TFLOPS incl. quantisation (4 H T^2 d per step)",
        "value": round(value, 2),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3+e8m0 (mxfp8) Q, K, V and softmax weights; fp32 softmax and accumulate; bf16 out",
        "data": "synthetic (seeded FLUX-shaped Q, K, V ~ N(0, 1))",
        "config": {"workload": f"flux_attention_{H}x{T}x{d}", "heads": H, "tokens": T, "head_dim": d,
                   "parallelism": f"replicas x{world}",
                   "step": "mxq_attention_mxfp8: MXFP8 of Q, K (per token) and V^T, one-pass softmax attention",
                   "l2": f"rotating {nsets} input sets ({nsets * 4 * H * T * d * 2 / 2**20:.0f} MiB > 126 MiB L2)"},
        "kernels_ms": {"step": round(step_ms, 5), "call_with_events": round(call_ms, 5)},
        "roofline": {"kernel": "attention_mxfp8_kernel + quantisers", "bound": "tensor",
                     "achieved": round(mma_flops / (step_ms * 1e-3) / 1e12, 2), "peak": round(peak, 1),
                     "unit": "TFLOP/s", "frac": round(mma_flops / (step_ms * 1e-3) / 1e12 / peak, 4),
                     "peak_kind": "burst",
                     "peak_source": f"{peaks['source']} bf16 burst x 2 (nominal fp8:bf16 dense ratio); "
                                    "achieved counts the 4 H T^2 d tensor-core flops of the step",
                     "traffic": None},
        "bf16_baseline": {"impl": "torch scaled_dot_product_attention, bf16, same tensors",
                          "value": round(whole_job_tflops(world, 1, flops, bf16_ms), 2), "unit": UNIT,
                          "ms_per_step": round(bf16_ms, 5), "speedup_of_value": round(bf16_ms / step_ms, 3)},
        "clocks": sampler.summary("headline"),
        "e2e": None,
        "gpu_launches": 4 * args.steps,
        "cpu_baseline": None,
    }


# ------------------------------------------------------------- CPU oracle
class OracleArm:
    """The oracle (as it stands) on the host cores.  Set-up, untimed: the
    workload's tensors, the weight's quantisation (offline, as on the GPU) and
    the activation's global amax (so that every sampled row is quantised
    exactly as in the full layer).  One step, timed: row chunks, each through
    the whole path -- its amax, its quantisation, the float64 GEMM -- until
    the step's time budget is spent (at least one chunk), continuing from
    where the previous step stopped and wrapping around the activation."""

    def __init__(self, workload: str):
        from oracle import gemm as G
        from oracle import quant as Q
        self.G, self.Q = G, Q
        self.case = workloads.make_case(workload)
        self.fmt = self.case.fmt
        if self.fmt == "nvfp4":
            qw = Q.quantize_nvfp4(self.case.W)
            self.Wd = Q.dequant_nvfp4(qw["codes"], qw["sf"], qw["g"])
        else:
            qw = Q.quantize_mxfp8(self.case.W)
            self.Wd = Q.dequant_mxfp8(qw["codes"], qw["sf"])
        self.amax = Q.amax(self.case.A) if self.fmt == "nvfp4" else None
        self.next_row = 0
        self.chunk = 64

    def step(self, budget_s: float):
        """Returns (rows processed, seconds)."""
        Q, G, case = self.Q, self.G, self.case
        self.chunk = 64 if budget_s >= 0.5 else 8
        rows = 0
        t0 = time.perf_counter()
        while rows == 0 or (time.perf_counter() - t0 < budget_s and rows < case.M):
            r0 = self.next_row
            a = case.A[r0:r0 + self.chunk]
            if self.fmt == "nvfp4":
                Q.amax(a)  # the chunk's share of the amax pass
                qa = Q.quantize_nvfp4(a, global_amax=self.amax)
                Ad = Q.dequant_nvfp4(qa["codes"], qa["sf"], qa["g"])
            else:
                qa = Q.quantize_mxfp8(a)
                Ad = Q.dequant_mxfp8(qa["codes"], qa["sf"])
            G.linear_ref(Ad, self.Wd, case.bias)
            rows += a.shape[0]
            self.next_row = (r0 + a.shape[0]) % case.M
        return rows, time.perf_counter() - t0

    def summary(self, rows: int, dt: float, steps: int):
        case = self.case
        try:
            threads = len(os.sched_getaffinity(0))
        except Exception:
            threads = os.cpu_count()
        return {
            "value": round(2.0 * rows * case.N * case.K / dt / 1e12, 6),
            "unit": UNIT,
            "cores": threads,
            "kind": "oracle",
            "sample": f"{steps} step(s) over {rows} rows of {case.name} ({case.M} rows, wrapping "
                      f"around): {self.chunk}-row chunks, each "
                      f"{'its amax, ' if self.fmt == 'nvfp4' else ''}{self.fmt} quantisation and "
                      f"float64 GEMM (Y and sum|ab|); {dt:.1f} s timed",
        }


def run_oracle_sample(workload: str, budget_s: float = 12.0):
    """The cpu_baseline leg: one bounded step of the oracle arm."""
    arm = OracleArm(workload)
    rows, dt = arm.step(budget_s)
    return arm.summary(rows, dt, 1)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--workload", default="c3", choices=["c1", "c2", "c3", "c4", "c5", "attn", "bf16", "mlp4"])
    ap.add_argument("--batch", type=int, default=1, choices=[1, 4],
                    help="batch of the c5 stack (1: 4608 tokens per image)")
    ap.add_argument("--impl", default="mxq", choices=["mxq", "reference"])
    ap.add_argument("--shape", default=None,
                    help="M,K,N of a seeded random layer instead of a named workload (profiling)")
    ap.add_argument("--fmt", default="nvfp4", choices=["nvfp4", "mxfp8"], help="format for --shape")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--min-dim", type=int, default=None,
                    help="selective-rule threshold (default 1024; c1 runs with 1, the NVFP4 path)")
    ap.add_argument("--no-tensor-scale", action="store_true",
                    help="NVFP4 without a per-tensor scale (g = 1 for weight and activation)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        # the CPU oracle on the host cores: rank 0 only, a few bounded samples
        if rank != 0:
            return 0
        if args.workload in ("c5", "attn", "bf16", "mlp4"):
            print(json.dumps({"impl": "reference", "unavailable": "the oracle arm times single "
                              "linear layers (c1-c4)"}))
            return 0
        # K timed steps after W untimed ones, each a bounded sample of the
        # workload sized so that the whole run stays within a few minutes
        arm = OracleArm(args.workload)
        budget = min(4.0, 100.0 / (args.steps + args.warmup))
        for _ in range(args.warmup):
            arm.step(budget)
        rows = 0
        dt = 0.0
        for _ in range(args.steps):
            r, t = arm.step(budget)
            rows += r
            dt += t
        sample = arm.summary(rows, dt, args.steps)
        value = sample["value"]
        out = {
            "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32 quantisation, f64 GEMM (CPU oracle)", "data": "synthetic",
            "config": {"workload": workloads.CASE_NAMES[args.workload]},
            "cpu_baseline": {"value": value, "unit": UNIT, "kind": sample["kind"],
                             "cores": sample["cores"], "sample": sample["sample"]},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
        }
        print(json.dumps(out))
        return 0

    dist = world > 1
    if dist:
        import datetime
        import torch.distributed as tdist
        torch.cuda.set_device(local_rank)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=torch.device("cuda", local_rank))
    try:
        if args.workload in ("c5", "attn", "bf16", "mlp4"):
            fn = {"c5": run_stack, "attn": run_attention, "bf16": run_bf16_branch, "mlp4": run_mlp}[args.workload]
            result = fn(args, rank, world, local_rank)
            if rank == 0:
                print(json.dumps(result))
            return 0
        result = run_gpu(args, rank, world, local_rank)
        if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.shape:
            result["cpu_baseline"] = run_oracle_sample(args.workload)
        if rank == 0:
            print(json.dumps(result))
    finally:
        if dist:
            import torch.distributed as tdist
            tdist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
