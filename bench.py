"""Benchmark: device-timed conv3d TFLOP/s on the video-VAE decoder workloads.

Default workload: bf16 256->256, 9x128x128 frames, 3x3x3 kernel, causal
replicate temporal padding, fused residual add (the 256-channel decoder block).
One step = one conv3d_fwd call over one synthetic batch (every stage of the
path: for this workload one kernel launch).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                  [--pass fwd|dgrad|wgrad] [--no-e2e] [--no-cpu-baseline] [--no-per-workload]

With the default workload the line also carries ``per_workload``: every other
decoder workload (cfg1, cfg3, cfg4, cfg5a-d) measured the same way in the same
process -- its own TFLOP/s, roofline, sampled parity against the oracle and
clocks.

Workloads: the convolutions cfg1..cfg5d, cfg2c (cached frames), cfg2s (stride), cfg4s, and the
GroupNorm + SiLU passes gn_cfg2, gn_cfg4.  --pass dgrad|wgrad times the backward passes of a
convolution workload (forward-equivalent FLOPs).  The roofline is tensor or HBM by the workload's
flop/B against the measured ridge point.

Multi-GPU (launched with torch.distributed.run): every rank convolves its own
seeded sample (data parallel over the batch, no data-path collective), so the
scaling is weak; value = FLOPs of all ranks / the slowest rank's time.
``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same
workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import seeded_inputs as si  # noqa: E402
from seeded_inputs.workloads import NORM_WORKLOADS, WORKLOADS  # noqa: E402

METRIC = "conv3d TFLOPS (bf16, video-VAE decoder shapes) and % of B200 dense peak"
TORCH_DTYPE = {"bf16": torch.bfloat16, "f16": torch.float16}
KERNEL_NAME = "conv3d_implicit_gemm_kernel"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SPEC_PEAKS = {"TFLOP/s": 2250.0, "GB/s": 8000.0}   # nominal dense bf16 and HBM3e (context only)


# ---------------------------------------------------------------- workload arithmetic

def out_shape(wl):
    kt, kh, kw = wl.kernel
    pt, ph, pw = wl.pad
    st, sh, sw = wl.stride
    pf, pb = (pt, pt) if wl.tpad == 0 else (kt - 1, 0)
    return ((wl.D + pf + pb - kt) // st + 1, (wl.H + 2 * ph - kh) // sh + 1,
            (wl.W + 2 * pw - kw) // sw + 1)


def algorithmic_flops(wl):
    """2 * Cout * Cin * kh * kw * sum over output pixels of the temporal taps that
    read a real frame (taps reading zero padding are not work).  A single causal
    replicate frame counts one folded temporal tap (the first-frame 2D conv)."""
    Do, Ho, Wo = out_shape(wl)
    kt, kh, kw = wl.kernel
    if wl.tpad == 1 and wl.D == 1:
        taps_t = Do * 1
    elif wl.tpad == 3:
        taps_t = Do * kt          # every tap reads a real (current or cached) frame
    else:
        pf = wl.pad[0] if wl.tpad == 0 else kt - 1
        taps_t = 0
        for to in range(Do):
            for it in range(kt):
                f = to * wl.stride[0] + it - pf
                if f < 0 and wl.tpad == 1:
                    f = 0
                taps_t += 0 <= f < wl.D
    return 2.0 * wl.N * Ho * Wo * wl.Cout * wl.Cin * kh * kw * taps_t


def algorithmic_bytes(wl):
    """x, w, bias, residual read once; y written once (16-bit elements)."""
    Do, Ho, Wo = out_shape(wl)
    x = wl.N * (wl.D + (wl.kernel[0] - 1 if wl.tpad == 3 else 0)) * wl.H * wl.W * wl.Cin
    w = wl.Cout * wl.kernel[0] * wl.kernel[1] * wl.kernel[2] * wl.Cin
    y = wl.N * Do * Ho * Wo * wl.Cout
    return 2.0 * (x + w + wl.Cout + y + (y if wl.residual else 0))


def nominal_flops(wl):
    """2 * M * N * K of the GEMM view (every tap counted, padding included)."""
    Do, Ho, Wo = out_shape(wl)
    return 2.0 * wl.N * Do * Ho * Wo * wl.Cout * wl.Cin * wl.kernel[0] * wl.kernel[1] * wl.kernel[2]


def describe(wl, world):
    Do, Ho, Wo = out_shape(wl)
    return {
        "workload": f"conv3d {wl.name}: {wl.note}",
        "dtype": wl.dtype, "N_per_gpu": wl.N, "global_batch": wl.N * world,
        "Cin": wl.Cin, "Cout": wl.Cout, "D": wl.D, "H": wl.H, "W": wl.W,
        "kernel": list(wl.kernel), "stride": list(wl.stride), "pad": list(wl.pad),
        "temporal_pad": ["zero", "causal_replicate", "causal_zero", "causal_cached"][wl.tpad],
        "residual": wl.residual, "out": [Do, Ho, Wo],
        "gemm": {"M": wl.N * Do * Ho * Wo, "N": wl.Cout,
                 "K": wl.Cin * wl.kernel[0] * wl.kernel[1] * wl.kernel[2]},
        "seed": wl.seed, "parallelism": f"dp{world}" if world > 1 else "single",
    }


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def kernel_source_hash():
    """Fingerprint of the device code the ncu counters were taken on."""
    h = hashlib.sha256()
    for rel in ("csrc/conv3d_kernel.cuh", "csrc/ptx.cuh"):
        with open(os.path.join(ROOT, "video_vae_convolution_implicit_b200", rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(wl_name):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(wl_name)
    if not e or e.get("kernel_sha") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- clocks (NVML, read only)

class ClockSampler:
    """Samples SM clock and clock-event reasons every ~5 ms while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index, label=None):
        # the timed region is also an NVTX range (`label`), so that profilers
        # can select it (ncu --nvtx --nvtx-include "<label>/")
        self.label = label
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = None
            try:  # CUDA and NVML number devices differently under CUDA_VISIBLE_DEVICES
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                self._h = pynvml.nvmlDeviceGetHandleByUUID(
                    uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception as e:  # no NVML: report null clocks
            self._err = str(e)
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(0.005)

    def _sample(self):
        try:
            self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
            mask = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            for bit, name in self.REASONS.items():
                if mask & bit and name != "gpu_idle":
                    self.reasons.add(name)
        except Exception:
            pass

    def __enter__(self):
        if self.label and torch.cuda.is_available():
            torch.cuda.nvtx.range_push(self.label)
        if self._ok:
            self._sample()
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._ok:
            self._stop.set()
            self._t.join()
            self._sample()
        if self.label and torch.cuda.is_available():
            torch.cuda.nvtx.range_pop()

    def summary(self):
        if not self._ok or not self.samples:
            return None
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": float(self.max_mhz),
                "sm_mhz_min": float(min(self.samples)), "reasons": sorted(self.reasons),
                "samples": len(self.samples), "sm_mhz_series": [int(v) for v in self.samples]}


# ---------------------------------------------------------------- oracle (CPU) timing

def host_bits(p):
    """16-bit patterns of the problem's tensors on the host (converted once)."""
    return {k: (None if p.get(k) is None else si.bits(p[k]))
            for k in ("x", "w", "bias", "residual", "prev")}


def oracle_rows_timed(hb, wl, rows):
    """The oracle on the given output pixels; returns (values, seconds of oracle work)."""
    import oracle
    t0 = time.perf_counter()
    ref = oracle.conv3d(hb["x"], hb["w"], hb["bias"], hb["residual"],
                        oracle.BF16 if wl.dtype == "bf16" else oracle.F16, wl.kernel, wl.stride,
                        wl.pad, wl.tpad, rows=rows, prev_bits=hb["prev"])
    return ref, time.perf_counter() - t0


def flops_per_row(wl):
    Do, Ho, Wo = out_shape(wl)
    return algorithmic_flops(wl) / (wl.N * Do * Ho * Wo)


def calibrated_rows(hb, wl, seconds, rng):
    """Number of output pixels the oracle finishes in about `seconds`."""
    Do, Ho, Wo = out_shape(wl)
    M = wl.N * Do * Ho * Wo
    n = 64
    while True:
        probe = np.sort(rng.choice(M, size=min(n, M), replace=False)).astype(np.int64)
        _, dt = oracle_rows_timed(hb, wl, probe)
        if dt > 0.5 or n >= M:
            break
        n *= 4
    per_row = max(dt / min(n, M), 1e-7)
    return int(max(16, min(M, seconds / per_row)))


def prev_frames(wl):
    return wl.kernel[0] - 1 if wl.tpad == 3 else 0


def host_problem(wl, seed):
    out = out_shape(wl)
    return si.conv3d_problem(wl.N, wl.Cin, wl.D, wl.H, wl.W, wl.Cout, wl.kernel, out, seed,
                             TORCH_DTYPE[wl.dtype], True, wl.residual, "cpu", prev_frames(wl))


def run_reference(args, wl, rank, world):
    """The reference arm: the fp64 CPU oracle as it stands, on a bounded sample."""
    if rank != 0:
        return 0
    import oracle
    hb = host_bits(host_problem(wl, wl.seed))
    Do, Ho, Wo = out_shape(wl)
    M = wl.N * Do * Ho * Wo
    rng = np.random.default_rng(wl.seed)
    budget = float(os.environ.get("CONV3D_REFERENCE_SECONDS", "90"))
    per_step_rows = calibrated_rows(hb, wl, budget / max(1, args.steps + args.warmup), rng)
    for _ in range(args.warmup):
        oracle_rows_timed(hb, wl, np.sort(rng.choice(M, per_step_rows, replace=False)))
    times = []
    for _ in range(args.steps):
        rows = np.sort(rng.choice(M, per_step_rows, replace=False)).astype(np.int64)
        _, dt = oracle_rows_timed(hb, wl, rows)
        times.append(dt)
    flops = flops_per_row(wl) * per_step_rows
    value = flops * len(times) / sum(times) / 1e12
    sample = (f"{per_step_rows} random output pixels (all {wl.Cout} channels) of {M} per step, "
              f"{args.steps} timed steps")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.mean(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": describe(wl, 1),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_reference_backward(args, wl, rank, world):
    """The reference arm of --pass dgrad|wgrad: the oracle's per-element adjoint sums as
    they stand, on a bounded random sample per step, scaled to forward-equivalent FLOPs
    by the sampled fraction of the elements."""
    if rank != 0:
        return 0
    import oracle
    Do, Ho, Wo = out_shape(wl)
    p = host_problem(wl, wl.seed)
    dy = si.tensor((wl.N, Do, Ho, Wo, wl.Cout), wl.seed, 5, 1.0, TORCH_DTYPE[wl.dtype], "cpu")
    hb, dyb = host_bits(p), si.bits(dy)
    flops = algorithmic_flops(wl)
    budget = float(os.environ.get("CONV3D_REFERENCE_SECONDS", "90")) / max(1, args.steps + args.warmup)
    n = 8
    while True:                                  # calibrate the sample to the per-step budget
        idx, total = _backward_samples(args.pass_, wl, n, 5)
        t0 = time.perf_counter()
        _oracle_backward_at(args.pass_, wl, hb, dyb, idx)
        dt = time.perf_counter() - t0
        if dt > budget / 4 or idx.size >= total:
            break
        n = int(n * min(16.0, max(2.0, budget / max(dt, 1e-3) / 2)))
    n = max(1, int(n * budget / max(dt, 1e-6))) if idx.size < total else n
    times, sizes = [], []
    for i in range(args.warmup + args.steps):
        idx, total = _backward_samples(args.pass_, wl, n, 100 + i)
        t0 = time.perf_counter()
        _oracle_backward_at(args.pass_, wl, hb, dyb, idx)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
            sizes.append(idx.size)
    value = flops * sum(sizes) / total / sum(times) / 1e12
    what = "input pixels (all channels) of dx" if args.pass_ == "dgrad" else "entries of dw"
    sample = (f"about {int(statistics.mean(sizes))} random {what} of {total} per step, "
              f"{args.steps} timed steps")
    line = {
        "impl": "reference", "metric": f"conv3d backward {args.pass_} TFLOPS (forward-equivalent FLOPs)",
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)", "config": dict(describe(wl, 1), direction=args.pass_),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- multi-rank plumbing

def rank_seed(wl, rank):
    """Each rank convolves its own independent sample (data parallel over the batch)."""
    return wl.seed + 1000 * rank


def max_over_ranks(value, device):
    """The slowest rank's time: MAX all-reduce (a timing collective, not a data path)."""
    if not torch.distributed.is_initialized() or torch.distributed.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(count, device):
    """A count summed over the ranks (SUM all-reduce; every rank takes part)."""
    if not torch.distributed.is_initialized() or torch.distributed.get_world_size() == 1:
        return int(count)
    t = torch.tensor([int(count)], dtype=torch.int64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return int(t.item())


def whole_job_tflops(flops_per_rank_step, world, steps, max_ms):
    """Units processed by all ranks divided by the slowest rank's time."""
    return flops_per_rank_step * world * steps / (max_ms * 1e-3) / 1e12


# ---------------------------------------------------------------- our arm

PER_WORKLOAD = ("cfg1", "cfg3", "cfg4", "cfg5a", "cfg5b", "cfg5c", "cfg5d")


def forward_launches(wl):
    """Library kernel launches per conv3d_fwd call: the main kernel, plus the
    first-frame fold for a single causal-replicate frame."""
    return 1 + (1 if (wl.tpad == 1 and wl.D == 1 and wl.kernel[0] > 1) else 0)


def roofline_for(flops, abytes, kernel_ms, peaks, peak_kind):
    """The roofline that bounds a workload: tensor above the ridge point, HBM below."""
    ridge = float(peaks["bf16_tflops"]) * 1e12 / (float(peaks["hbm_gbs"]) * 1e9)
    if flops / abytes >= ridge:
        roof = {"bound": "tensor", "achieved": flops / (kernel_ms * 1e-3) / 1e12,
                "peak": float(peaks["bf16_tflops"]), "unit": "TFLOP/s",
                "peak_source": f"{peak_kind} bf16_tflops (burst)"}
    else:
        roof = {"bound": "hbm", "achieved": abytes / (kernel_ms * 1e-3) / 1e9,
                "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                "peak_source": f"{peak_kind} hbm_gbs"}
    return dict(roof, frac=roof["achieved"] / roof["peak"],
                frac_of_spec=roof["achieved"] / SPEC_PEAKS[roof["unit"]],
                # long runs settle under the power cap: the measured sustained
                # cuBLAS figure is the matching denominator there
                frac_of_sustained=(roof["achieved"] / float(peaks["bf16_tflops_sustained"])
                                   if roof["bound"] == "tensor" and
                                   "bf16_tflops_sustained" in peaks else None),
                algorithmic_flops_per_launch=flops, algorithmic_bytes_per_launch=abytes,
                flop_per_byte=flops / abytes, ridge_flop_per_byte=ridge)


def measure_forward(args, wl, rank, world, local_rank, c3, keep=False):
    """One workload: seeded inputs on the device, warm-up, then args.steps
    conv3d_fwd calls, each bracketed by CUDA events on the launching stream
    with the L2 flushed in between; the slowest rank's total time.  Returns
    the measurement and (when `keep`) the problem tensors for the e2e leg."""
    dev = torch.device("cuda", local_rank)
    dt = TORCH_DTYPE[wl.dtype]
    Do, Ho, Wo = out_shape(wl)
    p = si.conv3d_problem(wl.N, wl.Cin, wl.D, wl.H, wl.W, wl.Cout, wl.kernel, (Do, Ho, Wo),
                          rank_seed(wl, rank), dt, True, wl.residual, dev, prev_frames(wl))
    y = torch.empty((wl.N, Do, Ho, Wo, wl.Cout), dtype=dt, device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(2 * l2 // 4 + 1024, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        c3.conv3d_fwd(p["x"], p["w"], p["bias"], p["residual"], y, wl.stride, wl.pad, wl.tpad,
                      stream=stream, prev=p["prev"])

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    if c3.poll_status(stream) != c3.Status.OK:
        raise RuntimeError(f"{wl.name}: device status after warm-up is not OK")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local_rank, f"timed {wl.name} fwd") as clocks:
        region0 = torch.cuda.Event(enable_timing=True)
        region1 = torch.cuda.Event(enable_timing=True)
        launches0 = c3.kernel_launches()
        region0.record(stream)
        for i in range(args.steps):
            flush.zero_()                       # L2 flushed between timed steps
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        region1.record(stream)
        launches1 = c3.kernel_launches()
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    max_ms = max_over_ranks(sum(step_ms), dev)
    status = c3.poll_status(stream)

    flops = algorithmic_flops(wl)
    peaks, peak_kind = load_peaks()
    # the dominant kernel's launch duration: the whole call's (for the first
    # frame the call also runs the short weight fold, so this is a lower bound)
    kernel_ms = statistics.mean(step_ms)
    abytes = algorithmic_bytes(wl)
    roof = roofline_for(flops, abytes, kernel_ms, peaks, peak_kind)
    roof.update(traffic=profiled_traffic(wl.name), kernel=KERNEL_NAME,
                timed=("whole call: the weight fold and the main kernel" if forward_launches(wl) > 1
                       else "the one kernel launch of the call"))
    res = {
        "value": whole_job_tflops(flops, world, args.steps, max_ms), "unit": "TFLOP/s",
        "ms_per_step": max_ms / args.steps,
        "roofline": roof,
        "nominal_tflops": whole_job_tflops(nominal_flops(wl), world, args.steps, max_ms),
        "algorithmic_gbs": abytes * world * args.steps / (max_ms * 1e-3) / 1e9,
        "gpu_launches": sum_over_ranks(launches1 - launches0, dev),
        "clocks": clocks.summary(),
        "step_ms": {"min": min(step_ms), "median": statistics.median(step_ms),
                    "p90": sorted(step_ms)[int(0.9 * (len(step_ms) - 1))], "max": max(step_ms),
                    "quarter_means": [statistics.mean(q) for q in
                                      (step_ms[i * len(step_ms) // 4:(i + 1) * len(step_ms) // 4]
                                       for i in range(4)) if q]},
        "region_ms": region0.elapsed_time(region1),
        "device_status": c3.status_string(status),
        "status_ok": status == c3.Status.OK,
    }
    if rank == 0:
        res["parity"] = parity_sample(wl, p, y)
    kept = (p, y, stream, dev, flops) if keep else None
    del flush
    return res, kept


def run_ours(args, wl, rank, world, local_rank):
    import video_vae_convolution_implicit_b200 as c3
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    res, (p, y, stream, dev, flops) = measure_forward(args, wl, rank, world, local_rank, c3,
                                                      keep=True)
    status_ok = res.pop("status_ok")
    line = {
        "metric": METRIC, "value": res["value"], "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": wl.dtype, "data": "synthetic (seeded SplitMix64 normals; no model weights)",
        "config": dict(describe(wl, world), l2="flushed (2x L2 write) between timed steps"),
    }
    line.update({k: v for k, v in res.items() if k not in ("value", "unit", "ms_per_step")})

    # end to end through the public API from pinned host buffers
    if not args.no_e2e:
        line["e2e"] = run_e2e(args, wl, p, y, stream, dev, c3, flops)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, p)
        line["speedup_over_oracle"] = line["value"] / line["cpu_baseline"]["value"]
    del p, y
    ok = status_ok and (rank != 0 or line["parity"]["ok"])

    # every other decoder workload, each measured the same way in this process
    if not args.no_per_workload and wl.name == "cfg2":
        per = {}
        for name in PER_WORKLOAD:
            other = WORKLOADS[name]
            r, _ = measure_forward(args, other, rank, world, local_rank, c3)
            r_ok = r.pop("status_ok")
            if r.get("clocks"):
                r["clocks"].pop("sm_mhz_series", None)
            r["config"] = describe(other, world)
            per[name] = r
            ok = ok and r_ok and (rank != 0 or r["parity"]["ok"])
            torch.cuda.empty_cache()
        line["per_workload"] = per

    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0 if ok else 1


def run_e2e(args, wl, p, y, stream, dev, c3, flops):
    """The same metric end to end from pinned host buffers: every step copies its
    inputs host -> device, runs conv3d_fwd through the C ABI and copies y back.
    Steps are pipelined over three streams with two device buffer sets, so step
    i+1's upload, step i's convolution and step i-1's download overlap (the
    copy engines and the SMs work at once); the bytes moved per step are those
    of one full step."""
    keys = ("x", "w", "bias", "residual", "prev")
    host = {k: (None if p[k] is None else p[k].cpu().pin_memory()) for k in keys}
    y_host = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(2)]
    dbuf = [{k: (None if p[k] is None else torch.empty_like(p[k])) for k in keys} for _ in range(2)]
    ybuf = [y, torch.empty_like(y)]
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = y_host[0].numel() * y_host[0].element_size()
    steps = max(2, min(args.steps, 20))
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    s_comp = stream
    ev = lambda: torch.cuda.Event()  # noqa: E731
    uploaded = [ev(), ev()]     # inputs of buffer set b are on the device
    consumed = [ev(), ev()]     # the conv using buffer set b has finished
    downloaded = [ev(), ev()]   # y of buffer set b has reached the host
    for b in range(2):
        consumed[b].record(s_comp)
        downloaded[b].record(s_out)

    def e2e_step(i):
        b = i % 2
        s_in.wait_event(consumed[b])
        with torch.cuda.stream(s_in):
            for k, v in host.items():
                if v is not None:
                    dbuf[b][k].copy_(v, non_blocking=True)
        uploaded[b].record(s_in)
        s_comp.wait_event(uploaded[b])
        s_comp.wait_event(downloaded[b])
        c3.conv3d_fwd(dbuf[b]["x"], dbuf[b]["w"], dbuf[b]["bias"], dbuf[b]["residual"], ybuf[b],
                      wl.stride, wl.pad, wl.tpad, stream=s_comp, prev=dbuf[b]["prev"])
        consumed[b].record(s_comp)
        s_out.wait_event(consumed[b])
        with torch.cuda.stream(s_out):
            y_host[b].copy_(ybuf[b], non_blocking=True)
        downloaded[b].record(s_out)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_in)
    for i in range(steps):
        e2e_step(i)
    s_in.wait_stream(s_out)
    end.record(s_in)
    torch.cuda.synchronize(dev)
    ms = start.elapsed_time(end) / steps
    # whole job: every rank's steps over the slowest rank's time (each rank ran
    # this leg, so the MAX reduction is a matching collective on all of them)
    world = torch.distributed.get_world_size() if torch.distributed.is_initialized() else 1
    max_ms = max_over_ranks(ms, dev)
    return {"value": whole_job_tflops(flops, world, 1, max_ms), "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d * world, "d2h_bytes_per_step": d2h * world,
            "ms_per_step": max_ms, "steps": steps, "ranks": world,
            "path": "pinned host -> device copies, conv3d_fwd (C ABI), device -> pinned host; "
                    "3 streams, 2 buffer sets (upload, compute and download of consecutive steps "
                    "overlap)"}


def _rows_for_parity(wl, n_random=48):
    Do, Ho, Wo = out_shape(wl)
    HoWo = Ho * Wo
    rows = set()
    for to in sorted({0, 1, Do - 1} & set(range(Do))):
        base = to * HoWo
        rows.update([base, base + Wo - 1, base + HoWo - 1, base + HoWo // 2])
    rng = np.random.default_rng(12345)
    rows.update(int(v) for v in rng.integers(0, wl.N * Do * HoWo, n_random))
    return np.array(sorted(rows), dtype=np.int64)


def parity_sample(wl, p, y):
    rows = _rows_for_parity(wl)
    ref, _ = oracle_rows_timed(host_bits(p), wl, rows)
    got = y.view(-1, wl.Cout)[torch.from_numpy(rows).to(y.device)].double().cpu().numpy()
    err = np.abs(got - ref)
    max_ratio = float(err.max() / np.abs(ref).max())
    rel_l1 = float(err.sum() / np.abs(ref).sum())
    # elementwise mean relative error, the denominator floored at 1e-3 max|ref| (reported only:
    # the bound is on the relative L1 form)
    floored = float(np.mean(err / np.maximum(np.abs(ref), 1e-3 * np.abs(ref).max())))
    return {"rows": int(rows.size), "max_err_over_max_ref": max_ratio, "rel_l1": rel_l1,
            "mean_rel_floored": floored,
            "ok": bool(np.isfinite(got).all() and max_ratio <= 1e-2 and rel_l1 <= 2e-3)}


def cpu_baseline(wl, p):
    """The oracle as it stands on a bounded random sample of the workload's
    output pixels (about CONV3D_CPU_BASELINE_SECONDS of CPU work)."""
    import oracle
    hb = host_bits(p)
    Do, Ho, Wo = out_shape(wl)
    M = wl.N * Do * Ho * Wo
    rng = np.random.default_rng(7)
    seconds = float(os.environ.get("CONV3D_CPU_BASELINE_SECONDS", "15"))
    n = calibrated_rows(hb, wl, seconds, rng)
    rows = np.sort(rng.choice(M, n, replace=False)).astype(np.int64)
    _, dt = oracle_rows_timed(hb, wl, rows)
    value = flops_per_row(wl) * n / dt / 1e12
    return {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n} random output pixels (all {wl.Cout} channels) of {M}, {dt:.1f} s"}


# ---------------------------------------------------------------- backward passes

def run_backward(args, wl, rank, world, local_rank):
    """dx (``--pass dgrad``) or dw + dbias (``--pass wgrad``) of one workload per
    step, through the C ABI.  Algorithmic FLOPs are the forward's: the backward
    passes form the same products.  One call launches several kernels (weight
    transform / clear, the tcgen05 GEMM, fold / conversion), so the roofline
    figure divides by the whole call's time and is a lower bound for the GEMM."""
    import video_vae_convolution_implicit_b200 as c3
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dt = TORCH_DTYPE[wl.dtype]
    Do, Ho, Wo = out_shape(wl)
    seed = rank_seed(wl, rank)
    p = si.conv3d_problem(wl.N, wl.Cin, wl.D, wl.H, wl.W, wl.Cout, wl.kernel, (Do, Ho, Wo), seed,
                          dt, True, False, dev)
    dy = si.tensor((wl.N, Do, Ho, Wo, wl.Cout), seed, 5, 1.0, dt, dev)
    x_shape = (wl.N, wl.D, wl.H, wl.W, wl.Cin)
    dtc = c3.BF16 if wl.dtype == "bf16" else c3.F16
    if args.pass_ == "dgrad":
        ws_bytes = c3.bwd_data_workspace_bytes(*x_shape[:1], wl.Cin, wl.D, wl.H, wl.W, wl.Cout,
                                               wl.kernel, wl.pad, wl.tpad)
        out = torch.empty(x_shape, dtype=dt, device=dev)
        db = None
    else:
        ws_bytes = c3.bwd_weight_workspace_bytes(wl.Cin, wl.Cout, wl.kernel)
        out = torch.empty((wl.Cout, *wl.kernel, wl.Cin), dtype=dt, device=dev)
        db = torch.empty((wl.Cout,), dtype=dt, device=dev)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(2 * l2 // 4 + 1024, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream

    def step():
        if args.pass_ == "dgrad":
            st = c3.conv3d_bwd_data_ptr(dy.data_ptr(), p["w"].data_ptr(), out.data_ptr(),
                                        *x_shape[:1], wl.Cin, wl.D, wl.H, wl.W, wl.Cout,
                                        wl.kernel, wl.stride, wl.pad, wl.tpad, dtc,
                                        ws.data_ptr(), ws.numel(), sh)
        else:
            st = c3.conv3d_bwd_weight_ptr(p["x"].data_ptr(), dy.data_ptr(), out.data_ptr(),
                                          db.data_ptr(), wl.N, wl.Cin, wl.D, wl.H, wl.W,
                                          wl.Cout, wl.kernel, wl.stride, wl.pad, wl.tpad, dtc,
                                          ws.data_ptr(), ws.numel(), sh)
        if st != c3.Status.OK:
            raise RuntimeError(f"backward call failed: {c3.status_string(st)}")

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    if c3.poll_status(stream) != c3.Status.OK:
        raise RuntimeError("device status after warm-up is not OK")
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local_rank, f"timed {wl.name} {args.pass_}") as clocks:
        launches0 = c3.kernel_launches()
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        launches = c3.kernel_launches() - launches0
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    max_ms = max_over_ranks(sum(step_ms), dev)
    status = c3.poll_status(stream)
    flops = algorithmic_flops(wl)
    value = whole_job_tflops(flops, world, args.steps, max_ms)
    peaks, peak_kind = load_peaks()
    call_ms = statistics.mean(step_ms)
    # algorithmic bytes: dgrad reads dy and w and writes dx; wgrad reads x and dy
    # and writes dw (+ dbias), all 16-bit
    x_el = wl.N * wl.D * wl.H * wl.W * wl.Cin
    y_el = wl.N * Do * Ho * Wo * wl.Cout
    w_el = wl.Cout * wl.kernel[0] * wl.kernel[1] * wl.kernel[2] * wl.Cin
    abytes = 2.0 * (y_el + w_el + x_el + (wl.Cout if args.pass_ == "wgrad" else 0))
    ridge = float(peaks["bf16_tflops"]) * 1e12 / (float(peaks["hbm_gbs"]) * 1e9)
    if flops / abytes >= ridge:
        roof = {"bound": "tensor", "achieved": flops / (call_ms * 1e-3) / 1e12,
                "peak": float(peaks["bf16_tflops"]), "unit": "TFLOP/s",
                "peak_source": f"{peak_kind} bf16_tflops (burst)"}
    else:
        roof = {"bound": "hbm", "achieved": abytes / (call_ms * 1e-3) / 1e9,
                "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                "peak_source": f"{peak_kind} hbm_gbs"}
    if args.pass_ == "dgrad":
        kernel = "conv3d_implicit_gemm_kernel (dgrad: transposed convolution of dy)"
    else:
        kernel = "conv3d_wgrad_kernel"
    line = {
        "metric": f"conv3d backward {args.pass_} TFLOPS (forward-equivalent FLOPs)",
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype,
        "data": "synthetic (seeded SplitMix64 normals; dy stream 5)",
        "config": dict(describe(wl, world), direction=args.pass_, residual=False,
                       l2="flushed (2x L2 write) between timed steps"),
        "roofline": dict(roof, frac=roof["achieved"] / roof["peak"],
                         frac_of_spec=roof["achieved"] / SPEC_PEAKS[roof["unit"]], traffic=None,
                         kernel=kernel,
                         timed="whole call (all its launches): a lower bound for the GEMM",
                         algorithmic_flops_per_launch=flops, algorithmic_bytes_per_launch=abytes,
                         flop_per_byte=flops / abytes, ridge_flop_per_byte=ridge),
        "nominal_tflops": whole_job_tflops(nominal_flops(wl), world, args.steps, max_ms),
        "gpu_launches": sum_over_ranks(launches, dev),
        "clocks": clocks.summary(),
        "step_ms": {"min": min(step_ms), "median": statistics.median(step_ms),
                    "p90": sorted(step_ms)[int(0.9 * (len(step_ms) - 1))], "max": max(step_ms)},
        "device_status": c3.status_string(status),
    }
    if rank == 0:
        line["parity"] = backward_parity(args.pass_, wl, p, dy, out, db)
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = backward_cpu_baseline(args.pass_, wl, p, dy, flops)
            line["speedup_over_oracle"] = value / line["cpu_baseline"]["value"]
        print(json.dumps(line), flush=True)
    ok = status == c3.Status.OK and (rank != 0 or line["parity"]["ok"])
    return 0 if ok else 1


def _backward_samples(which, wl, n, seed):
    rng = np.random.default_rng(seed)
    if which == "dgrad":
        total = wl.N * wl.D * wl.H * wl.W
        fixed = [0, wl.W - 1, wl.H * wl.W - 1, total - 1]      # corners, first / last frame
    else:
        total = wl.Cout * wl.kernel[0] * wl.kernel[1] * wl.kernel[2] * wl.Cin
        fixed = [0, total - 1]
    idx = set(fixed) | {int(v) for v in rng.integers(0, total, n)}
    return np.array(sorted(idx), dtype=np.int64), total


def _oracle_backward_at(which, wl, hb, dy_bits, idx):
    import oracle
    dt = oracle.BF16 if wl.dtype == "bf16" else oracle.F16
    if which == "dgrad":
        return oracle.conv3d_dx_at(hb["w"], dy_bits, dt, (wl.N, wl.D, wl.H, wl.W, wl.Cin),
                                   wl.kernel, wl.stride, wl.pad, wl.tpad, idx)
    return oracle.conv3d_dw_at(hb["x"], dy_bits, dt, wl.Cout, wl.kernel, wl.stride, wl.pad,
                               wl.tpad, idx)


def backward_parity(which, wl, p, dy, out, db):
    """Sampled elements of dx (whole pixels, all channels) or dw (single
    entries) and the whole dbias against the oracle's per-element sums."""
    hb = host_bits(p)
    dyb = si.bits(dy)
    if which == "dgrad":
        n = 48
    else:   # each dw entry sums over every output pixel: keep the oracle to ~5e8 products
        Do, Ho, Wo = out_shape(wl)
        n = int(min(256, max(32, 5e8 / (wl.N * Do * Ho * Wo))))
    idx, _ = _backward_samples(which, wl, n, 4321)
    ref = _oracle_backward_at(which, wl, hb, dyb, idx)
    flat = out.view(-1, wl.Cin) if which == "dgrad" else out.view(-1)
    got = flat[torch.from_numpy(idx).to(out.device)].double().cpu().numpy()
    errs = [np.abs(got - ref)]
    refs = [ref]
    if db is not None:
        import oracle
        ref_db = oracle.decode16(dyb, oracle.BF16 if wl.dtype == "bf16" else oracle.F16)
        ref_db = ref_db.reshape(-1, wl.Cout).sum(axis=0)
        errs.append(np.abs(db.double().cpu().numpy() - ref_db))
        refs.append(ref_db)
    res = {"samples": int(idx.size), "what": "dx pixels" if which == "dgrad" else "dw entries"}
    ok = bool(np.isfinite(got).all())
    for name, e, r in zip(("", "dbias_"), errs, refs):
        mr = float(e.max() / np.abs(r).max())
        rl = float(e.sum() / np.abs(r).sum())
        res[name + "max_err_over_max_ref"] = mr
        res[name + "rel_l1"] = rl
        ok = ok and mr <= 1e-2 and rl <= 2e-3
    res["ok"] = ok
    return res


def backward_cpu_baseline(which, wl, p, dy, flops):
    """The oracle's per-element sums on a bounded random sample, scaled to FLOPs
    by the sampled fraction of the elements (every element of dw, or every
    pixel of dx, carries on average total/elements of the work)."""
    import oracle
    hb = host_bits(p)
    dyb = si.bits(dy)
    seconds = float(os.environ.get("CONV3D_CPU_BASELINE_SECONDS", "15"))
    n = 16
    while True:
        idx, total = _backward_samples(which, wl, n, 99)
        t0 = time.perf_counter()
        _oracle_backward_at(which, wl, hb, dyb, idx)
        dt = time.perf_counter() - t0
        if dt > seconds / 4 or idx.size >= total:
            break
        n = int(n * min(16.0, max(2.0, seconds / max(dt, 1e-3) / 2)))
    value = flops * idx.size / total / dt / 1e12
    what = "input pixels (all channels) of dx" if which == "dgrad" else "entries of dw"
    return {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{idx.size} random {what} of {total}, {dt:.1f} s"}


# ---------------------------------------------------------------- GroupNorm + SiLU workloads

def run_norm(args, wl, rank, world, local_rank):
    """GroupNorm statistics + fused normalise/SiLU over one activation tensor per
    step: HBM-bound (x read twice, y written once)."""
    import oracle
    import video_vae_convolution_implicit_b200 as c3
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    td = TORCH_DTYPE[wl.dtype]
    N, D, H, W, C = wl.shape
    seed = wl.seed + 1000 * rank
    x = si.tensor(wl.shape, seed, 0, 1.0, td, dev)
    gamma = (si.tensor((C,), seed, 1, 0.2, torch.float32, dev) + 1.0).to(td)
    beta = si.tensor((C,), seed, 2, 0.2, td, dev)
    y = torch.empty_like(x)
    sets = N * D if wl.per_frame else N
    stats = torch.empty((sets, wl.groups, 2), dtype=torch.float64, device=dev)
    flush = torch.empty(2 * torch.cuda.get_device_properties(dev).L2_cache_size // 4 + 1024,
                        dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        c3.groupnorm_stats(x, wl.groups, 1e-6, wl.per_frame, stats, stream)
        if ev:
            ev[1].record(stream)
        c3.groupnorm_silu(x, stats, gamma, beta, y, wl.groups, wl.per_frame, True, stream)
        if ev:
            ev[2].record(stream)

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local_rank, f"timed {wl.name} groupnorm") as clocks:
        launches0 = c3.kernel_launches()
        for i in range(args.steps):
            flush.zero_()
            step(evs[i])
        launches = c3.kernel_launches() - launches0
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    stats_ms = [e[0].elapsed_time(e[1]) for e in evs]
    apply_ms = [e[1].elapsed_time(e[2]) for e in evs]
    my_ms = sum(a + b for a, b in zip(stats_ms, apply_ms))
    max_ms = max_over_ranks(my_ms, dev)
    tensor_bytes = x.numel() * x.element_size()
    step_bytes = 3 * tensor_bytes
    value = step_bytes * world * args.steps / (max_ms * 1e-3) / 1e9
    peaks, peak_kind = load_peaks()
    peak = float(peaks["hbm_gbs"])
    apply_gbs = 2 * tensor_bytes / (statistics.mean(apply_ms) * 1e-3) / 1e9
    stats_gbs = tensor_bytes / (statistics.mean(stats_ms) * 1e-3) / 1e9
    line = {
        "metric": "GroupNorm+SiLU HBM GB/s (x read twice, y written once)", "value": value,
        "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": max_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic (seeded SplitMix64 normals)",
        "config": {"workload": f"{wl.name}: {wl.note}", "shape_ndhwc": list(wl.shape),
                   "groups": wl.groups, "per_frame": wl.per_frame, "global_batch": N * world,
                   "l2": "flushed (2x L2 write) between timed steps"},
        "roofline": {"bound": "hbm", "achieved": apply_gbs, "peak": peak, "unit": "GB/s",
                     "frac": apply_gbs / peak, "traffic": None,
                     "peak_source": f"{peak_kind} hbm_gbs", "kernel": "gn_apply_kernel",
                     "algorithmic_bytes_per_launch": 2 * tensor_bytes,
                     "stats_kernel_gbs": stats_gbs, "stats_kernel_frac": stats_gbs / peak},
        "gpu_launches": sum_over_ranks(launches, dev),
        "clocks": clocks.summary(),
    }
    if rank == 0:
        # parity gate: the oracle on the whole tensor (or on whole frames when the
        # statistics are per frame)
        if wl.per_frame:
            frames = sorted({0, D - 1})
            xs = x[:, frames].contiguous()
            got = y[:, frames].double().cpu().numpy()
        else:
            xs = x
            got = y.double().cpu().numpy()
        ref = oracle.groupnorm_silu(si.bits(xs), si.bits(gamma), si.bits(beta),
                                    oracle.BF16 if wl.dtype == "bf16" else oracle.F16, wl.groups,
                                    eps=1e-6, per_frame=wl.per_frame)
        err = np.abs(got - ref)
        mr = float(err.max() / np.abs(ref).max())
        rl = float(err.sum() / np.abs(ref).sum())
        line["parity"] = {"elements": int(ref.size), "max_err_over_max_ref": mr, "rel_l1": rl,
                          "ok": bool(np.isfinite(got).all() and mr <= 1e-2 and rl <= 2e-3)}
        print(json.dumps(line), flush=True)
    return 0 if rank != 0 or line["parity"]["ok"] else 1


# ---------------------------------------------------------------- decoder block: GroupNorm + SiLU + conv

def run_gnblock(args, wl, rank, world, local_rank):
    """One decoder block (GroupNorm(32) + SiLU, then the workload's convolution)
    timed four ways on the same inputs: `separate` = statistics pass, apply
    pass (writes h) and conv3d_fwd(h); `apply_conv_stats` = apply pass and a
    convolution that gathers the GroupNorm statistics of its own output (what
    the next block needs), this block's statistics coming from the previous
    block's; `fused` = statistics pass and conv3d_fwd_gn with the transform in
    the operand path (h never written); `chained` = the operand-path form that
    also gathers its output's statistics.  value = the fastest form's TFLOP/s
    (conv FLOPs over the block's time); every form is parity-gated on sampled
    rows against the oracle composition (GroupNorm + SiLU in fp64, one
    rounding, fp64 conv)."""
    import oracle
    import video_vae_convolution_implicit_b200 as c3
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    td = TORCH_DTYPE[wl.dtype]
    Do, Ho, Wo = out_shape(wl)
    G = 32
    seed = rank_seed(wl, rank)
    p = si.conv3d_problem(wl.N, wl.Cin, wl.D, wl.H, wl.W, wl.Cout, wl.kernel, (Do, Ho, Wo), seed,
                          td, True, wl.residual, dev)
    x = p["x"]
    gamma = (si.tensor((wl.Cin,), seed, 6, 0.2, torch.float32, dev) + 1.0).to(td)
    beta = si.tensor((wl.Cin,), seed, 7, 0.2, td, dev)
    h = torch.empty_like(x)
    y = torch.empty((wl.N, Do, Ho, Wo, wl.Cout), dtype=td, device=dev)
    stats = torch.empty((wl.N, G, 2), dtype=torch.float64, device=dev)
    flush = torch.empty(2 * torch.cuda.get_device_properties(dev).L2_cache_size // 4 + 1024,
                        dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    kw = dict(stride=wl.stride, pad=wl.pad, tpad=wl.tpad, stream=stream)

    def separate():
        c3.groupnorm_stats(x, G, 1e-6, False, stats, stream)
        c3.groupnorm_silu(x, stats, gamma, beta, h, G, False, True, stream)
        c3.conv3d_fwd(h, p["w"], p["bias"], p["residual"], y, wl.stride, wl.pad, wl.tpad,
                      stream=stream)

    def fused():
        c3.groupnorm_stats(x, G, 1e-6, False, stats, stream)
        c3.conv3d_gn(x, stats, gamma, beta, p["w"], p["bias"], p["residual"], y, G, **kw)

    def chained():
        c3.conv3d_gn(x, stats, gamma, beta, p["w"], p["bias"], p["residual"], y, G,
                     out_groups=G, **kw)

    def apply_conv_stats():
        # this block's statistics come from the previous block's epilogue; the
        # convolution gathers the next block's in its own
        c3.groupnorm_silu(x, stats, gamma, beta, h, G, False, True, stream)
        c3.conv3d_gn(h, None, None, None, p["w"], p["bias"], p["residual"], y, out_groups=G,
                     **kw)

    # the parts on their own, to decompose the forms
    def stats_only():
        c3.groupnorm_stats(x, G, 1e-6, False, stats, stream)

    def apply_only():
        c3.groupnorm_silu(x, stats, gamma, beta, h, G, False, True, stream)

    def conv_only():
        c3.conv3d_fwd(h, p["w"], p["bias"], p["residual"], y, wl.stride, wl.pad, wl.tpad,
                      stream=stream)

    def conv_stats_only():
        c3.conv3d_gn(h, None, None, None, p["w"], p["bias"], p["residual"], y, out_groups=G,
                     **kw)

    forms = {"separate": separate, "apply_conv_stats": apply_conv_stats, "fused": fused,
             "chained": chained}
    parts = {"stats": stats_only, "apply": apply_only, "conv": conv_only,
             "conv_with_stats": conv_stats_only}
    flops = algorithmic_flops(wl)
    res = {}
    if rank == 0:
        # the oracle's h: GroupNorm + SiLU in fp64, rounded once (as an unfused pipeline stores it)
        hbits = si.bits(torch.from_numpy(oracle.groupnorm_silu(
            si.bits(x), si.bits(gamma), si.bits(beta),
            oracle.BF16 if wl.dtype == "bf16" else oracle.F16, G, eps=1e-6)).to(td))
        hb = dict(host_bits(p), x=hbits)
        rows = _rows_for_parity(wl)
    for name, fn in forms.items():
        for _ in range(max(3, args.warmup)):
            flush.zero_()
            fn()
        torch.cuda.synchronize(dev)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        if world > 1:
            torch.distributed.barrier()
        with ClockSampler(local_rank, f"timed {wl.name} block {name}") as clocks:
            launches0 = c3.kernel_launches()
            for a, b in ev:
                flush.zero_()
                a.record(stream)
                fn()
                b.record(stream)
            launches = c3.kernel_launches() - launches0
            torch.cuda.synchronize(dev)
        ms = [a.elapsed_time(b) for a, b in ev]
        max_ms = max_over_ranks(sum(ms), dev)
        st = c3.poll_status(stream)
        r = {"ms_per_step": max_ms / args.steps,
             "tflops": whole_job_tflops(flops, world, args.steps, max_ms),
             "gpu_launches": sum_over_ranks(launches, dev), "device_status": c3.status_string(st),
             "clocks": clocks.summary()}
        if r["clocks"]:
            r["clocks"].pop("sm_mhz_series", None)
        if rank == 0:
            ref, _ = oracle_rows_timed(hb, wl, rows)
            got = y.view(-1, wl.Cout)[torch.from_numpy(rows).to(dev)].double().cpu().numpy()
            err = np.abs(got - ref)
            mr, rl = float(err.max() / np.abs(ref).max()), float(err.sum() / np.abs(ref).sum())
            r["parity"] = {"rows": int(rows.size), "max_err_over_max_ref": mr, "rel_l1": rl,
                           "ok": bool(np.isfinite(got).all() and mr <= 1e-2 and rl <= 2e-3)}
        res[name] = r
    part_ms = {}
    for name, fn in parts.items():
        for _ in range(max(3, args.warmup)):
            flush.zero_()
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        for a, b in ev:
            flush.zero_()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize(dev)
        part_ms[name] = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), dev) / args.steps
    peaks, peak_kind = load_peaks()
    best = min(res, key=lambda k: res[k]["ms_per_step"])
    conv_roof = roofline_for(flops, algorithmic_bytes(wl), res[best]["ms_per_step"], peaks,
                             peak_kind)
    line = {
        "metric": "decoder block (GroupNorm+SiLU -> conv3d) TFLOPS, conv FLOPs over the block's time",
        "value": res[best]["tflops"], "unit": "TFLOP/s", "n_gpus": world, "best_form": best,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": res[best]["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype,
        "data": "synthetic (seeded SplitMix64 normals)",
        "config": dict(describe(wl, world), groupnorm_groups=G, l2="flushed between steps"),
        "roofline": dict(conv_roof, kernel=KERNEL_NAME, timed="the whole block (every launch)"),
        "forms": res,
        "parts_ms": part_ms,
        "gpu_launches": res[best]["gpu_launches"],
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    ok = all(r["device_status"] == "ok" and (rank != 0 or r["parity"]["ok"]) for r in res.values())
    return 0 if ok else 1


# ---------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="cfg2", choices=sorted(WORKLOADS) + sorted(NORM_WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--pass", dest="pass_", default="fwd",
                    choices=["fwd", "dgrad", "wgrad", "gnblock"],
                    help="forward convolution (default), one of its backward passes, or the "
                         "decoder block GroupNorm+SiLU -> conv in its separate and fused forms")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="with the default workload, skip the other decoder workloads")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    is_norm = args.workload in NORM_WORKLOADS
    wl = NORM_WORKLOADS[args.workload] if is_norm else WORKLOADS[args.workload]

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and world > 1:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)

    if args.impl == "reference":
        if is_norm:
            print(json.dumps({"impl": "reference", "unavailable":
                              "the reference arm times the convolution oracle only"}))
            return 0
        if args.pass_ == "gnblock":
            print(json.dumps({"impl": "reference", "unavailable":
                              "the reference arm times the convolution oracle only"}))
            return 0
        if args.pass_ != "fwd":
            return run_reference_backward(args, wl, rank, world)
        return run_reference(args, wl, rank, world)

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        if is_norm:
            fn = run_norm
        elif args.pass_ == "gnblock":
            fn = run_gnblock
        else:
            fn = run_ours if args.pass_ == "fwd" else run_backward
        rc = fn(args, wl, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    return rc


if __name__ == "__main__":
    sys.exit(main())
