#!/usr/bin/env python
"""Benchmark of the exact IO-aware attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload c3]

One step is one pass of the whole path over one batch of synthetic input: the
forward (O and LSE) and the backward (D, recomputation with dK/dV/dQ
accumulation, dQ conversion). The default workload is B=2, H=32, N=8192,
d=128, causal, bf16. It is the shape on which the pages' long-context claims
and the forward/backward utilisation targets are stated (N >= 8K, d = 128,
forward and backward). FLOPs are algorithmic: 4 B H N^2 d for the forward,
halved for causal; 2.5x that for the backward.

Rank 0 prints one JSON line. `value` is the whole-job TFLOP/s over all ranks
(weak scaling: every rank runs its own replica of the workload; there is no
data-path collective). `e2e` repeats the measurement with each step's inputs
copied from pinned host memory and the results copied back inside the timed
region. `roofline` reports the dominant kernel against the measured dense bf16
peak. `cpu_baseline` times the float64 oracle on a bounded sample on the host
cores. `--impl reference` times that oracle alone as the reference arm.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention fwd/bwd TFLOP/s on 1 B200 and % of dense BF16 tensor peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
# fp32 on the CUDA cores (the fp32 forward's roofline): 148 SMs x 128 fp32 lanes x 2 FLOP
# per FMA x the 1965 MHz maximum SM clock, a nominal figure (no fp32 peak is measured)
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
L2_BYTES = 126 << 20

# DRAM bytes (read + write) per launch of the dominant kernel from one ncu
# capture, with the hash of the kernel source it was taken on. A changed
# source makes the figure stale and the bench reports null.
NCU_TRAFFIC = {
    # profiles/bwd_main_d128_B2H32N8192_causal.md
    ("bwd_main", "c3"): {"bytes_per_launch": 810053376 + 491489280, "csrc_sha": "5f1ce705a7c0333f"},
    # profiles/bwd_main_d64_B4H16N2048_causal.md
    ("bwd_main", "c2"): {"bytes_per_launch": 101773056 + 22512384, "csrc_sha": "ca60193791cdd550"},
    # profiles/fwd_bf16_d128_B2H32N8192_causal.md, profiles/fwd_bf16_d256_B2H16N8192_causal.md
    ("fwd", "c3"): {"bytes_per_launch": 403569664 + 117326848, "csrc_sha": "d22978f98dcad723"},
    ("fwd", "c4"): {"bytes_per_launch": 809743360 + 260787968, "csrc_sha": "d22978f98dcad723"},
    ("fwd", "c6"): {"bytes_per_launch": 403493888 + 118081024, "csrc_sha": "b1a823b364771c18"},
    # profiles/decode_B16Hq32Hkv8_Nk32768_d128.md, profiles/decode_wide_B16Hq64Hkv8Nq8_Nk32768_d128.md
    ("decode_split", "dec"): {"bytes_per_launch": 2148206592 + 3491072, "csrc_sha": "d4b94526a7290b64"},
    ("decode_split", "dec4"): {"bytes_per_launch": 1074812160 + 4385280, "csrc_sha": "d4b94526a7290b64"},
    ("decode_split", "dec8"): {"bytes_per_launch": 2153774592 + 7643648, "csrc_sha": "d4b94526a7290b64"},
    ("decode_split", "dec64"): {"bytes_per_launch": 1074049792 + 3947520, "csrc_sha": "d4b94526a7290b64"},
}


# The source text each kernel is built from: its own definition (start marker up
# to end marker) plus the shared device helpers. Edits elsewhere in the file (the
# other head-dim variant, comments) leave the recorded counters valid.
KERNEL_SOURCES = {
    "bwd_main": ("fa_bwd_sm100.cu", [("#ifndef FA_BWD_POLY_PAIRS", "// Register split: the launch gives"),
                                     ("__device__ __forceinline__ void red_add(", "// ----"),
                                     ("struct Bwd128Cfg {", "struct Bwd64Cfg {")]),
    "bwd_main_d64": ("fa_bwd_sm100.cu", [("#ifndef FA_BWD_POLY_PAIRS", "// Register split: the launch gives"),
                                         ("struct Bwd64Cfg {", "template <int D>\ncudaError_t launch_preprocess_d(")]),
    "fwd": ("fa_fwd_sm100.cu", [("constexpr int kFwdThreads = 384;", "// fwd256_kernel (bf16")]),
    "fwd256": ("fa_fwd_sm100.cu", [("constexpr int kFwdThreads = 384;", "template <int D, bool FP8>\nstruct FwdCfg {"),
                                   ("struct FwdUnit {", "// PERSIST: the grid"),
                                   ("// fwd256_kernel (bf16", "template <int D, int KIND>\ncudaError_t launch_fwd_d(")]),
    "decode_split": ("fa_decode_sm100.cu", [("template <int R>\nstruct DecCfg {", "template <int R>\ncudaError_t launch_decode_r(")]),
}


def kernel_source_hash(kernel: str) -> str:
    fname, spans = KERNEL_SOURCES[kernel]
    csrc = os.path.join(ROOT, "exact_io_aware_44_b200", "csrc")
    h = hashlib.sha256()
    with open(os.path.join(csrc, fname)) as f:
        text = f.read()
    for start, end in spans:
        a = text.index(start) if start else 0
        b = text.index(end, a) if end else len(text)
        h.update(text[a:b].encode())
    with open(os.path.join(csrc, "sm100.cuh"), "rb") as f:
        h.update(f.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# ranks
# ---------------------------------------------------------------------------

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(value: float, group=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    backend = dist.get_backend(group)
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else torch.device("cpu")
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def barrier(group=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier(group=group)


def job_throughput(flops_per_step_per_rank: float, world: int, max_seconds_per_step: float) -> float:
    """Whole-job TFLOP/s: every rank's work over the slowest rank's time."""
    return flops_per_step_per_rank * world / max_seconds_per_step / 1e12


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    """SM clock, power and clock-event reasons sampled every `interval_ms` by a
    host thread through NVML while the timed region runs. `mark(True)` /
    `mark(False)` bracket the region; the summary uses the samples inside it
    (falling back to all samples when the region is shorter than one period).
    Without NVML it falls back to `nvidia-smi -lms`. It only reads settings."""

    REASONS = (("sw_power_cap", 0x4), ("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20),
               ("hw_thermal_slowdown", 0x40), ("hw_power_brake_slowdown", 0x80))

    def __init__(self, cuda_index: int, interval_ms: int = 10):
        self.cuda_index = cuda_index
        self.interval = interval_ms / 1000.0
        self.samples = []      # (t, sm_mhz, max_mhz, power_w, reasons bitmask)
        self.window = [None, None]
        self._stop = None
        self._thread = None
        self._smi = None
        self._nv = None  # (module, handle, reasons function, max SM clock) once NVML is up

    def _handle(self, nv):
        import torch
        try:
            uuid = str(torch.cuda.get_device_properties(self.cuda_index).uuid)
            return nv.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def _sample(self):
        """One NVML reading (clock, max clock, power, reasons) appended to the samples."""
        nv, h, reasons_fn, mx = self._nv
        try:
            self.samples.append((time.perf_counter(), nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), mx,
                                 nv.nvmlDeviceGetPowerUsage(h) / 1000.0, int(reasons_fn(h))))
        except Exception:
            pass

    def _poll(self):
        while not self._stop.is_set():
            self._sample()
            self._stop.wait(self.interval)

    def __enter__(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._handle(nv)
            reasons_fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            self._nv = (nv, h, reasons_fn, nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self._stop = threading.Event()
            self._thread = threading.Thread(target=self._poll, daemon=True)
            self._thread.start()
        except Exception:
            self._thread = None
            self._nv = None
            self._start_smi()
        time.sleep(0.05)
        return self

    def _start_smi(self):
        fields = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.sw_power_cap,"
                  "clocks_event_reasons.hw_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                  "clocks_event_reasons.hw_thermal_slowdown")
        fd, path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self._smi = (subprocess.Popen(["nvidia-smi", f"--id={self.cuda_index}", f"--query-gpu={fields}",
                                           "--format=csv,noheader,nounits", "-lms=20"],
                                          stdout=open(path, "w"), stderr=subprocess.DEVNULL), path)
        except OSError:
            self._smi = None

    def mark(self, start: bool):
        """Bracket the timed region; with NVML, a reading is taken at each edge too, so that a
        region shorter than the polling interval still has samples of its own."""
        if start:
            self.window[0] = time.perf_counter()
        if self._nv is not None:
            self._sample()
        if not start:
            self.window[1] = time.perf_counter()

    def __exit__(self, *exc):
        time.sleep(0.02)
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
        if self._smi is not None:
            proc, path = self._smi
            proc.terminate()
            try:
                proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                proc.kill()
            for r in csv.reader(io.StringIO(open(path).read())):
                try:
                    bits = sum(bit for (name, bit), val in zip(self.REASONS[:4], r[3:7])
                               if val.strip().lower() == "active")
                    self.samples.append((None, float(r[0]), float(r[1]), float(r[2]), bits))
                except (ValueError, IndexError):
                    continue
            os.unlink(path)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock samples"]}
        t0, t1 = self.window
        inside = [s for s in self.samples if s[0] is not None and t0 is not None and t1 is not None
                  and t0 <= s[0] <= t1]
        used = inside if len(inside) >= 3 else self.samples
        sm = [s[1] for s in used]
        reasons = sorted({name for s in used for name, bit in self.REASONS if s[4] & bit})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(s[2] for s in used), "sm_mhz_min": min(sm),
                "reasons": reasons, "samples": len(used),
                "window": "timed region" if used is inside else "whole sampler run (region shorter than 3 periods)",
                "interval_ms": round(self.interval * 1000), "power_w_max": max(s[3] for s in used),
                "source": "nvml" if self._thread is not None else "nvidia-smi"}


# ---------------------------------------------------------------------------
# CPU baseline: the float64 oracle on a bounded sample of the workload
# ---------------------------------------------------------------------------

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_head_step(w, b: int, h: int):
    """Forward (+ backward) of one (batch, head) of workload `w` in float64; returns (seconds, FLOPs)."""
    import numpy as np
    import oracle
    import synth
    ds = w.descale if w.dtype in ("e4m3", "e5m2") else 1.0  # FP8 slices hold codes; real value = code * descale
    q = synth.head_slice(w, synth.TID_Q, b, h)[None, None].astype(np.float64) * ds
    k = synth.head_slice(w, synth.TID_K, b, h // w.group)[None, None].astype(np.float64) * ds
    v = synth.head_slice(w, synth.TID_V, b, h // w.group)[None, None].astype(np.float64) * ds
    do = synth.head_slice(w, synth.TID_DO, b, h)[None, None] if w.backward else None
    t0 = time.perf_counter()
    o, lse = oracle.attention_fwd64(q, k, v, w.causal, w.scale)
    if w.backward:
        oracle.attention_bwd64(q, k, v, do, w.causal, w.scale, o=o, lse=lse)
    dt = time.perf_counter() - t0
    f = 4.0 * w.N * w.N * w.d * (0.5 if w.causal else 1.0)
    return dt, f * (3.5 if w.backward else 1.0)


def cpu_baseline(w, budget_s: float = 15.0):
    total_t, total_f, heads = 0.0, 0.0, 0
    while heads < w.B * w.Hq and (heads == 0 or total_t < budget_s):
        b, h = divmod(heads, w.Hq)
        dt, f = oracle_head_step(w, b, h)
        total_t += dt
        total_f += f
        heads += 1
    what = "forward + backward" if w.backward else "forward"
    full_f = (w.fwd_flops() + (w.bwd_flops() if w.backward else 0.0))
    return {"value": total_f / total_t / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "full_problem_seconds_extrapolated": round(full_f / (total_f / total_t), 1),
            "sample": f"{heads} of {w.B * w.Hq} (batch, head) pairs, full {what} each, float64 NumPy",
            "seconds": round(total_t, 3)}


# ---------------------------------------------------------------------------
# our path
# ---------------------------------------------------------------------------

def run_ours(args, w, world, rank, local):
    import numpy as np
    import torch

    import exact_io_aware_44_b200 as fa
    import synth

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    fp8 = w.dtype in ("e4m3", "e5m2")
    e5m2 = w.dtype == "e5m2"
    f32 = w.dtype == "f32"  # the fp32 forward on the CUDA cores
    # dense FP8 peak = measured bf16 x the nominal 2x (4.5 vs 2.25 PFLOP/s dense)
    peak_mul = 2.0 if fp8 else 1.0
    peak = FP32_ALU_TFLOPS if f32 else float(peaks["bf16_tflops"]) * peak_mul
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, args.cpu_budget)

    # inputs: generated on the host (seeded), kept pinned for the e2e leg
    host = {}
    tids = (("q", synth.TID_Q), ("k", synth.TID_K), ("v", synth.TID_V)) + ((("do", synth.TID_DO),) if w.backward else ())
    in_dtype = ((torch.float8_e5m2 if e5m2 else torch.float8_e4m3fn) if fp8
                else torch.float32 if f32 else torch.bfloat16)
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.N, w.d
    share = 1.0
    if args.shard == "heads":
        # strong scaling: this rank computes its slice of the flattened head axis
        q0, q1, k0, k1 = fa.head_shard(B, Hq, Hkv, rank, world)
        share = (k1 - k0) / (B * Hkv)
    for name, tid in tids:
        x = synth.tensor(w, tid)
        if args.shard == "heads":
            lo, hi = (q0, q1) if name in ("q", "do") else (k0, k1)
            x = x.reshape(B * x.shape[1], N, d)[lo:hi][None]
        host[name] = torch.from_numpy(np.ascontiguousarray(x)).to(in_dtype).pin_memory()
    d_in = {n: t.to(dev) for n, t in host.items()}
    if args.shard == "heads":
        B, Hq, Hkv = 1, q1 - q0, k1 - k0
    o = torch.empty((B, Hq, N, d), dtype=torch.float32 if f32 else torch.bfloat16, device=dev)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=dev)
    # Inputs and outputs smaller than L2 would stay cached from one step to the next: then a
    # buffer larger than L2 is overwritten before every timed step, outside the step's events.
    step_bytes = sum(t.numel() * t.element_size() for t in d_in.values()) + o.numel() * o.element_size()
    if w.backward:
        step_bytes += o.numel() * o.element_size() * 2 + (B * Hkv * N * d * 2) * 2
    l2_flush = torch.empty(4 * L2_BYTES, dtype=torch.uint8, device=dev) if step_bytes < 2 * L2_BYTES else None
    if w.backward:
        dq = torch.empty_like(o)
        dk = torch.empty((B, Hkv, N, d), dtype=torch.bfloat16, device=dev)
        dv = torch.empty_like(dk)
        ws = torch.empty(fa.workspace_bytes(B, Hq, Hkv, N, d), dtype=torch.uint8, device=dev)
    P = lambda t: t.data_ptr()

    def step(events=None):
        if events is not None:
            events[0].record(stream)
        if fp8:
            ds = w.descale
            rc = fa.fwd_fp8_raw(P(d_in["q"]), P(d_in["k"]), P(d_in["v"]), ds, ds, ds, P(o), P(lse), B, Hq, Hkv, N, d,
                                w.causal, w.scale, sp, e5m2=e5m2)
        else:
            rc = fa.fwd_raw(P(d_in["q"]), P(d_in["k"]), P(d_in["v"]), P(o), P(lse), B, Hq, Hkv, N, d, w.causal,
                            w.scale, sp, f32=f32)
        if rc:
            raise fa.FAError(rc, "fa_fwd_fp8" if fp8 else "fa_fwd_f32" if f32 else "fa_fwd")
        if not w.backward:
            if events is not None:
                for e in events[1:]:
                    e.record(stream)
            return
        between = None
        if events is not None:
            between = lambda i: events[1 + i].record(stream)
        rc = fa.bwd_phases_raw(P(d_in["q"]), P(d_in["k"]), P(d_in["v"]), P(o), P(lse), P(d_in["do"]), P(dq), P(dk),
                               P(dv), P(ws), B, Hq, Hkv, N, d, w.causal, w.scale, sp, between=between)
        if rc:
            raise fa.FAError(rc, "fa_bwd")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = fa.get_status()
    if st:
        raise fa.FAError(st, "warm-up")

    # ---------------------------------------------------- device-timed region
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(K)]
    with ClockSampler(local) as clocks:
        barrier()
        torch.cuda.synchronize()
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        clocks.mark(True)
        t_start.record(stream)
        for i in range(K):
            if l2_flush is not None:
                l2_flush.fill_(i & 0xFF)
            step(evs[i])
        t_end.record(stream)
        torch.cuda.synchronize()
        clocks.mark(False)
        barrier()
    st = fa.get_status()
    if st:
        raise fa.FAError(st, "timed region")
    ms_total = t_start.elapsed_time(t_end)
    if l2_flush is not None:  # the steps' own spans, without the overwrites between them
        ms_total = sum(e[0].elapsed_time(e[4]) for e in evs)
    ms_step = reduce_max(ms_total / K)
    # events: 0 fwd start, 1 bwd pre start (= fwd end), 2 main start, 3 convert start, 4 bwd end
    per_kernel = {name: [e[i].elapsed_time(e[i + 1]) for e in evs]
                  for i, name in enumerate(("fwd", "bwd_preprocess", "bwd_main", "bwd_convert"))}
    fwd_ms, pre_ms, main_ms, conv_ms = (statistics.mean(per_kernel[n]) for n in per_kernel)
    f_fwd, f_bwd = w.fwd_flops() * share, (w.bwd_flops() * share if w.backward else 0.0)
    if args.shard == "heads":  # the ranks' shares add up to one workload
        value = (w.fwd_flops() + (w.bwd_flops() if w.backward else 0.0)) / (ms_step / 1e3) / 1e12
    else:
        value = job_throughput(f_fwd + f_bwd, world, ms_step / 1e3)

    kernels = {
        "fwd": {"ms": fwd_ms, "tflops": f_fwd / fwd_ms / 1e9},
        "bwd_preprocess": {"ms": pre_ms},
        "bwd_main": {"ms": main_ms, "tflops": f_bwd / main_ms / 1e9 if main_ms > 0 else 0.0},
        "bwd_convert": {"ms": conv_ms},
    }
    dominant = max(("fwd", "bwd_main"), key=lambda k: kernels[k]["ms"])
    achieved = kernels[dominant]["tflops"]
    dom_ms_med = statistics.median(per_kernel[dominant])
    achieved_med = (f_fwd if dominant == "fwd" else f_bwd) / dom_ms_med / 1e9
    traffic = None
    src_name = ("bwd_main_d64" if (dominant == "bwd_main" and d == 64)
                else "fwd256" if (dominant == "fwd" and d == 256) else dominant)
    rec = NCU_TRAFFIC.get((dominant, w.name))
    if rec and rec.get("csrc_sha") == kernel_source_hash(src_name):
        traffic = rec["bytes_per_launch"]
    roofline = {"bound": "alu" if f32 else "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": UNIT,
                "frac": round(achieved / peak, 4), "traffic": traffic, "kernel": dominant,
                "peak_source": ("nominal fp32 FMA rate: 148 SMs x 128 lanes x 2 FLOP x 1965 MHz" if f32 else
                                (f"{peak_src} dense bf16 burst (MEASURED_PEAKS.json bf16_tflops)"
                                 if peak_src == "measured" else "fallback 1.59 PFLOP/s")
                                + (" x 2, the nominal dense fp8:bf16 ratio" if fp8 else "")),
                "frac_of_sustained": round(achieved / (float(peaks.get("bf16_tflops_sustained", peak)) * peak_mul),
                                           4),
                # achieved/frac above use the mean launch time over the timed steps; these the median
                "achieved_median": round(achieved_med, 1), "frac_median": round(achieved_med / peak, 4)}

    # ---------------------------------------------------- end to end (host buffers)
    # Through the public C ABI, every step uploads its inputs from pinned host memory
    # and downloads its results. Two device buffer sets let step i's kernels overlap
    # step i+1's upload and step i-1's download, each on its own stream (copies in
    # both directions run alongside the kernels), as a user of the API would run it.
    # The serial variant (copy in, compute, copy out on one stream) is reported too.
    e2e = None
    if not args.no_e2e:
        dev_out = {"o": o, "lse": lse}
        if w.backward:
            dev_out.update(dq=dq, dk=dk, dv=dv)
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = sum(t.numel() * t.element_size() for t in dev_out.values())
        Ke = max(1, min(K, args.e2e_steps))
        flops_job = ((w.fwd_flops() + (w.bwd_flops() if w.backward else 0.0)) if args.shard == "heads" else None)

        def user_step(ins, outs, wsb, sptr):
            if fp8:
                ds = w.descale
                rc = fa.fwd_fp8_raw(P(ins["q"]), P(ins["k"]), P(ins["v"]), ds, ds, ds, P(outs["o"]), P(outs["lse"]),
                                    B, Hq, Hkv, N, d, w.causal, w.scale, sptr, e5m2=e5m2)
            else:
                rc = fa.fwd_raw(P(ins["q"]), P(ins["k"]), P(ins["v"]), P(outs["o"]), P(outs["lse"]), B, Hq, Hkv, N,
                                d, w.causal, w.scale, sptr, f32=f32)
            if rc:
                raise fa.FAError(rc, "fa_fwd")
            if w.backward:
                rc = fa.bwd_raw(P(ins["q"]), P(ins["k"]), P(ins["v"]), P(outs["o"]), P(outs["lse"]), P(ins["do"]),
                                P(outs["dq"]), P(outs["dk"]), P(outs["dv"]), P(wsb), B, Hq, Hkv, N, d, w.causal,
                                w.scale, sptr)
                if rc:
                    raise fa.FAError(rc, "fa_bwd")

        def rate(ms):
            if flops_job is not None:
                return flops_job / (ms / 1e3) / 1e12
            return job_throughput(f_fwd + f_bwd, world, ms / 1e3)

        # serial: one stream
        out_host0 = {n: torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for n, t in dev_out.items()}
        barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(Ke):
            for n in host:
                d_in[n].copy_(host[n], non_blocking=True)
            user_step(d_in, dev_out, ws if w.backward else None, sp)
            for n in out_host0:
                out_host0[n].copy_(dev_out[n], non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        serial_ms = reduce_max(e0.elapsed_time(e1) / Ke)

        # overlapped: two buffer sets, upload / compute / download streams
        sets = [(d_in, dev_out, ws if w.backward else None, out_host0),
                ({n: torch.empty_like(t) for n, t in d_in.items()},
                 {n: torch.empty_like(t) for n, t in dev_out.items()},
                 torch.empty_like(ws) if w.backward else None,
                 {n: torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for n, t in dev_out.items()})]
        s_up, s_down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        up_done = [torch.cuda.Event() for _ in range(2)]
        comp_done = [torch.cuda.Event() for _ in range(2)]
        down_done = [torch.cuda.Event() for _ in range(2)]
        barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s_up)
        for i in range(Ke):
            bi = i % 2
            ins, outs, wsb, hout = sets[bi]
            if i >= 2:
                s_up.wait_event(comp_done[bi])     # step i-2's kernels are done with this set's inputs
            with torch.cuda.stream(s_up):
                for n in host:
                    ins[n].copy_(host[n], non_blocking=True)
            up_done[bi].record(s_up)
            stream.wait_event(up_done[bi])
            if i >= 2:
                stream.wait_event(down_done[bi])   # step i-2's results have left this set's outputs
            user_step(ins, outs, wsb, sp)
            comp_done[bi].record(stream)
            s_down.wait_event(comp_done[bi])
            with torch.cuda.stream(s_down):
                for n in hout:
                    hout[n].copy_(outs[n], non_blocking=True)
            down_done[bi].record(s_down)
        for ev in down_done:
            stream.wait_event(ev)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e_ms = reduce_max(e0.elapsed_time(e1) / Ke)
        e2e = {"value": round(rate(e_ms), 2), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e_ms, 3),
               "steps": Ke, "overlap": "upload, kernels and download of consecutive steps on three streams",
               "serial": {"value": round(rate(serial_ms), 2), "ms_per_step": round(serial_ms, 3)}}
        st = fa.get_status()
        if st:
            raise fa.FAError(st, "e2e region")

    clk = clocks.summary()
    result = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
        "scaling": "strong" if args.shard == "heads" else "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": f"{w.name}: B={B} Hq={Hq} Hkv={Hkv} N={N} d={d} "
                               f"{'causal' if w.causal else 'non-causal'} {w.dtype} "
                               f"{'fwd+bwd' if w.backward else 'fwd'}",
                   "B": B, "Hq": Hq, "Hkv": Hkv, "N": N, "d": d, "causal": w.causal,
                   "l2": ("inputs larger than L2 ("
                          + ("Q, K, V, O, dO are" if w.backward else "Q, K, V are")
                          + f" {B * Hq * N * d * (1 if fp8 else 4 if f32 else 2) / 1e6:.0f} MB each; L2 is 126 MB)"
                          if l2_flush is None else
                          f"L2 flushed: a {4 * L2_BYTES >> 20} MB buffer is overwritten before every timed step "
                          f"(the step's tensors, {step_bytes / 1e6:.1f} MB, would fit in the 126 MB L2); the step "
                          "time sums the steps' own event spans, without the overwrites"),
                   "parallelism": f"head shards x{world}" if args.shard == "heads" else f"replicas x{world}"},
        "pct_of_peak": round(100 * value / world / peak, 2),
        "fwd_tflops": round(kernels["fwd"]["tflops"], 1),
        "bwd_tflops": round(f_bwd / (pre_ms + main_ms + conv_ms) / 1e9, 1) if w.backward else None,
        "kernels_ms": {k: round(v["ms"], 4) for k, v in kernels.items()},
        "kernels_ms_median_min": {k: [round(statistics.median(v), 4), round(min(v), 4)]
                                  for k, v in per_kernel.items() if (w.backward or k == "fwd")},
        # first timed step and slowest step per kernel: where a mean above the median comes from
        "kernels_ms_first_max": {k: [round(v[0], 4), round(max(v), 4)]
                                 for k, v in per_kernel.items() if (w.backward or k == "fwd")},
        # The pages' traffic argument: standard attention writes the N x N scores and
        # reads them back (fp16 S and P, each written and read once: 8 B*Hq*N^2 bytes);
        # this path moves only the O(N) tensors (algorithmic bytes; ncu-measured DRAM
        # bytes of the dominant kernel in `roofline.traffic`).
        "traffic_model": {"standard_attention_bytes": 8 * B * Hq * N * N,
                          # Q, K, V read (input dtype), O written (bf16; fp32 for fp32 inputs), LSE written (fp32)
                          "fwd_algorithmic_bytes": (B * Hq + 2 * B * Hkv) * N * d * (1 if fp8 else 4 if f32 else 2)
                          + B * Hq * N * d * (4 if f32 else 2) + B * Hq * N * 4,
                          "bwd_workspace_bytes": fa.workspace_bytes(B, Hq, Hkv, N, d) if w.backward else 0,
                          "note": "the workspace is linear in N (D and the fp32 dQ accumulator); "
                                  "no N x N buffer exists"},
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": (4 if w.backward else 1) * K,
        "clocks": clk,
    }
    if w.name == "c3" and world == 1 and args.shard != "heads" and not args.no_extras:
        result["other_configs"] = other_configs(args, fa, torch, dev, stream, peak)
    return result


def other_configs(args, fa, torch, dev, stream, peak):
    """The remaining workloads the utilisation targets name, timed after the main
    line on the same device: the c4 forward, the c5 forward and backward, the c2
    (d = 64) forward and backward, three decode steps (dec, dec8, dec64), and the d = 256
    forward (c6). Same timing as the main line: CUDA events around each launch on the
    launching stream, after warm-up, no parity work inside. Inputs: c4, c5, c6 and decode
    are drawn on the device by a
    seeded torch generator with the workloads' distributions (iid N(0, 1)), since
    they are larger than L2 and drawing them on the host would dominate the run;
    c2 uses the parity tests' seeded host recipe (with its spiked rows) and, being
    smaller than L2, a 512 MB buffer is overwritten before every timed launch."""
    import synth
    sp = stream.cuda_stream
    P = lambda t: t.data_ptr()
    K = max(5, min(args.steps, 20))
    Wm = max(3, args.warmup)
    gen = torch.Generator(device=dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    peaks_all, _ = load_peaks()
    peak_sustained = float(peaks_all.get("bf16_tflops_sustained", peak))
    out = {}

    last_clocks = {}

    def timed(launches, n_events, l2_flush):
        """Run `launches(events)` Wm + K times; returns per-interval lists of ms. The
        clocks seen during the K timed runs are left in last_clocks."""
        for _ in range(Wm):
            launches(None)
        torch.cuda.synchronize()
        rec = []
        with ClockSampler(dev.index if dev.index is not None else 0) as clocks:
            clocks.mark(True)
            for _ in range(K):
                if l2_flush:
                    flush.fill_(1)
                evs = [torch.cuda.Event(enable_timing=True) for _ in range(n_events)]
                launches(evs)
                rec.append(evs)
            torch.cuda.synchronize()
            clocks.mark(False)
        last_clocks.clear()
        last_clocks.update(clocks.summary())
        st = fa.get_status()
        if st:
            raise fa.FAError(st, "other configs")
        return [[r[i].elapsed_time(r[i + 1]) for r in rec] for i in range(n_events - 1)]

    def entry(wname, shape, ms_lists, names, f_fwd, f_bwd, inputs):
        e = {"shape": shape, "inputs": inputs, "steps": K, "warmup": Wm,
             "clocks": {k: last_clocks.get(k) for k in ("sm_mhz", "sm_mhz_min", "reasons", "samples")}}
        med = {n: statistics.median(v) for n, v in zip(names, ms_lists)}
        e["ms_median"] = {n: round(v, 4) for n, v in med.items()}
        e["fwd_tflops"] = round(f_fwd / med["fwd"] / 1e9, 1)
        e["fwd_pct_of_peak"] = round(100 * f_fwd / med["fwd"] / 1e9 / peak, 2)
        if f_bwd:
            bwd_ms = med["bwd_preprocess"] + med["bwd_main"] + med["bwd_convert"]
            e["bwd_tflops"] = round(f_bwd / bwd_ms / 1e9, 1)
            e["bwd_pct_of_peak"] = round(100 * f_bwd / bwd_ms / 1e9 / peak, 2)
            e["bwd_main_tflops"] = round(f_bwd / med["bwd_main"] / 1e9, 1)
            e["bwd_main_frac"] = round(f_bwd / med["bwd_main"] / 1e9 / peak, 4)
            e["bwd_main_frac_of_sustained"] = round(f_bwd / med["bwd_main"] / 1e9 / peak_sustained, 4)
        e["fwd_frac_of_sustained"] = round(f_fwd / med["fwd"] / 1e9 / peak_sustained, 4)
        out[wname] = e

    def attn(wl, tensors, inputs, l2_flush):
        B, Hq, Hkv, N, d = wl.B, wl.Hq, wl.Hkv, wl.N, wl.d
        q, k, v = tensors[:3]
        o = torch.empty((B, Hq, N, d), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=dev)
        if wl.backward:
            do = tensors[3]
            dq, dk, dv = torch.empty_like(o), torch.empty_like(k), torch.empty_like(v)
            ws = torch.empty(fa.workspace_bytes(B, Hq, Hkv, N, d), dtype=torch.uint8, device=dev)

        def launches(evs):
            if evs is not None:
                evs[0].record(stream)
            rc = fa.fwd_raw(P(q), P(k), P(v), P(o), P(lse), B, Hq, Hkv, N, d, wl.causal, wl.scale, sp)
            if rc:
                raise fa.FAError(rc, "fa_fwd")
            if evs is not None:
                evs[1].record(stream)
            if wl.backward:
                between = (lambda i: evs[1 + i].record(stream)) if evs is not None else None
                rc = fa.bwd_phases_raw(P(q), P(k), P(v), P(o), P(lse), P(do), P(dq), P(dk), P(dv), P(ws), B, Hq,
                                       Hkv, N, d, wl.causal, wl.scale, sp, between=between)
                if rc:
                    raise fa.FAError(rc, "fa_bwd")

        names = ("fwd", "bwd_preprocess", "bwd_main", "bwd_convert") if wl.backward else ("fwd",)
        ms = timed(launches, len(names) + 1, l2_flush)
        shape = (f"B={B} Hq={Hq} Hkv={Hkv} N={N} d={d} {'causal' if wl.causal else 'non-causal'} bf16 "
                 f"{'fwd+bwd' if wl.backward else 'fwd'}")
        entry(wl.name, shape, ms, names, wl.fwd_flops(), wl.bwd_flops() if wl.backward else 0.0, inputs)

    def dev_randn(wl, tid, heads):
        gen.manual_seed(wl.seed * 16 + tid)
        x = torch.randn((wl.B, heads, wl.N, wl.d), generator=gen, device=dev, dtype=torch.float32)
        return (x * wl.std).to(torch.bfloat16)

    for name in ("c4", "c5", "c6"):
        wl = synth.WORKLOADS[name]
        ts = [dev_randn(wl, tid, wl.Hq if tid in (synth.TID_Q, synth.TID_DO) else wl.Hkv)
              for tid in ((synth.TID_Q, synth.TID_K, synth.TID_V) + ((synth.TID_DO,) if wl.backward else ()))]
        attn(wl, ts, "seeded torch.randn on the device, iid N(0,1), rounded to bf16", False)
        del ts
    wl = synth.WORKLOADS["c2"]
    ts = [torch.from_numpy(synth.tensor(wl, tid)).to(dev, torch.bfloat16)
          for tid in (synth.TID_Q, synth.TID_K, synth.TID_V, synth.TID_DO)]
    attn(wl, ts, "the parity tests' seeded host recipe (1% of query rows x20); L2 overwritten before each step",
         True)
    del ts
    # decode: one new query per head against a 32768-key cache (dec, 4 query rows a group), and
    # eight new tokens per sequence of a 64-head model (dec8, 64 query rows a group), and the
    # first at a head dim of 64 (dec64)
    for dname in ("dec", "dec8", "dec64"):
        dw = synth.DECODE_WORKLOADS[dname]
        gen.manual_seed(dw.seed)
        qd = torch.randn((dw.B, dw.Hq, dw.Nq, dw.d), generator=gen, device=dev).to(torch.bfloat16)
        kd = torch.randn((dw.B, dw.Hkv, dw.Nk, dw.d), generator=gen, device=dev).to(torch.bfloat16)
        vd = torch.randn((dw.B, dw.Hkv, dw.Nk, dw.d), generator=gen, device=dev).to(torch.bfloat16)
        od = torch.empty_like(qd)
        ld = torch.empty((dw.B, dw.Hq, dw.Nq), dtype=torch.float32, device=dev)
        wsd = torch.empty(fa.decode_workspace_bytes(dw.B, dw.Hq, dw.Hkv, dw.Nq, dw.Nk, dw.d), dtype=torch.uint8,
                          device=dev)

        def dec_launch(evs):
            if evs is not None:
                evs[0].record(stream)
            rc = fa.decode_raw(P(qd), P(kd), P(vd), P(od), P(ld), P(wsd), dw.B, dw.Hq, dw.Hkv, dw.Nq, dw.Nk, dw.d,
                               dw.causal, dw.scale, 0, sp)
            if rc:
                raise fa.FAError(rc, "fa_decode")
            if evs is not None:
                evs[1].record(stream)

        ms = statistics.median(timed(dec_launch, 2, False)[0])
        peaks, _ = load_peaks()
        algo = dw.kv_bytes() + 2 * qd.numel() * 2 + ld.numel() * 4
        out[dname] = {"shape": f"decode B={dw.B} Hq={dw.Hq} Hkv={dw.Hkv} Nq={dw.Nq} Nk={dw.Nk} d={dw.d} causal bf16",
                      "inputs": "seeded torch.randn on the device, iid N(0,1), rounded to bf16",
                      "ms_median": round(ms, 4), "gbs": round(algo / ms / 1e6, 1),
                      "frac_of_hbm": round(algo / ms / 1e6 / float(peaks["hbm_gbs"]), 4), "steps": K, "warmup": Wm,
                      "clocks": {k: last_clocks.get(k) for k in ("sm_mhz", "sm_mhz_min", "reasons", "samples")}}
        del qd, kd, vd, od, ld, wsd
    del flush
    return out


# ---------------------------------------------------------------------------
# decode workload (one new query per head against a long K/V cache)
# ---------------------------------------------------------------------------

DECODE_METRIC = "attention decode: K/V cache bytes read per second on 1 B200 (% of measured HBM bandwidth)"


def oracle_decode_head(w, q, k, v, b, h):
    import numpy as np
    import oracle
    kvh = h // w.group
    t0 = time.perf_counter()
    oracle.decode_fwd64(q[b:b + 1, h:h + 1].astype(np.float64), k[b:b + 1, kvh:kvh + 1], v[b:b + 1, kvh:kvh + 1],
                        w.causal, w.scale)
    return time.perf_counter() - t0


def run_decode(args, w, world, rank, local):
    import torch

    import exact_io_aware_44_b200 as fa
    import synth

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    q, k, v = synth.decode_inputs(w)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        heads, tot = 0, 0.0
        while heads < w.B * w.Hq and (heads == 0 or tot < args.cpu_budget):
            b, h = divmod(heads, w.Hq)
            tot += oracle_decode_head(w, q, k, v, b, h)
            heads += 1
        per_head_bytes = 2 * w.Nk * w.d * 2
        cpu = {"value": round(heads * per_head_bytes / tot / 1e9, 3), "unit": "GB/s", "cores": blas_threads(),
               "kind": "oracle", "sample": f"{heads} of {w.B * w.Hq} query heads, float64 NumPy (each head reads "
                                           f"its kv head's cache)", "seconds": round(tot, 3)}
    host_q = torch.from_numpy(q).to(torch.bfloat16).pin_memory()
    dq = host_q.to(dev)
    dk = torch.from_numpy(k).to(torch.bfloat16).to(dev)
    dv = torch.from_numpy(v).to(torch.bfloat16).to(dev)
    del k, v
    o = torch.empty_like(dq)
    lse = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=dev)
    ws = torch.empty(fa.decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d), dtype=torch.uint8, device=dev)
    P = lambda t: t.data_ptr()

    def step():
        rc = fa.decode_raw(P(dq), P(dk), P(dv), P(o), P(lse), P(ws), w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal,
                           w.scale, 0, sp)
        if rc:
            raise fa.FAError(rc, "fa_decode")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if fa.get_status():
        raise fa.FAError(fa.get_status(), "warm-up")
    K = args.steps
    with ClockSampler(local) as clocks:
        barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        clocks.mark(True)
        e0.record(stream)
        for _ in range(K):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        clocks.mark(False)
        barrier()
    if fa.get_status():
        raise fa.FAError(fa.get_status(), "timed region")
    ms = reduce_max(e0.elapsed_time(e1) / K)
    kv_bytes = w.kv_bytes()
    rec = NCU_TRAFFIC.get(("decode_split", w.name))
    traffic = rec["bytes_per_launch"] if rec and rec.get("csrc_sha") == kernel_source_hash("decode_split") else None
    algo_bytes = kv_bytes + 2 * dq.numel() * 2 + lse.numel() * 4  # K, V read; q read, o written; lse
    gbs = algo_bytes / (ms / 1e3) / 1e9
    value = world * gbs
    e2e = None
    if not args.no_e2e:  # the cache stays on the device; each step brings its queries and returns o, lse
        out_o = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        out_l = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
        Ke = max(1, min(K, args.e2e_steps))
        barrier()
        torch.cuda.synchronize()
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(Ke):
            dq.copy_(host_q, non_blocking=True)
            step()
            out_o.copy_(o, non_blocking=True)
            out_l.copy_(lse, non_blocking=True)
        a1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e_ms = reduce_max(a0.elapsed_time(a1) / Ke)
        e2e = {"value": round(world * algo_bytes / (e_ms / 1e3) / 1e9, 1), "unit": "GB/s",
               "h2d_bytes_per_step": host_q.numel() * 2, "d2h_bytes_per_step": out_o.numel() * 2 + out_l.numel() * 4,
               "ms_per_step": round(e_ms, 4), "steps": Ke}
    return {
        "metric": DECODE_METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{w.name}: decode B={w.B} Hq={w.Hq} Hkv={w.Hkv} Nq={w.Nq} Nk={w.Nk} d={w.d} "
                               f"{'causal' if w.causal else 'non-causal'} bf16",
                   "l2": f"inputs larger than L2 (K and V caches {kv_bytes / 1e9:.2f} GB; L2 is 126 MB)",
                   "parallelism": f"replicas x{world}"},
        "tflops": round(w.flops() / (ms / 1e3) / 1e12, 2),
        "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                     "frac": round(gbs / hbm, 4), "traffic": traffic, "kernel": "decode_split+merge",
                     "peak_source": f"{peak_src} HBM copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": 2 * K,  # the split kernel and the merge
        "clocks": clocks.summary(),
    }


# ---------------------------------------------------------------------------
# reference arm: the float64 oracle as it stands, on the host cores
# ---------------------------------------------------------------------------

def run_reference(args, w):
    times, flops = [], 0.0
    n_heads = w.B * w.Hq
    for i in range(args.warmup + args.steps):
        b, h = divmod(i % n_heads, w.Hq)
        dt, f = oracle_head_step(w, b, h)
        if i >= args.warmup:
            times.append(dt)
            flops = f
    ms = 1e3 * statistics.mean(times)
    value = flops / (ms / 1e3) / 1e12
    what = "forward + backward" if w.backward else "forward"
    sample = f"one (batch, head) pair per step: full {what} of B=1 H=1 N={w.N} d={w.d} in float64"
    return {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": 0, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{w.name}: B={w.B} Hq={w.Hq} Hkv={w.Hkv} N={w.N} d={w.d} "
                                   f"{'causal' if w.causal else 'non-causal'} {w.dtype} "
                                   f"{'fwd+bwd' if w.backward else 'fwd'} (sampled per step)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "kind": "oracle", "cores": blas_threads(),
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_reference_decode(args, w):
    import synth
    q, k, v = synth.decode_inputs(w)
    times = []
    for i in range(args.warmup + args.steps):
        b, h = divmod(i % (w.B * w.Hq), w.Hq)
        dt = oracle_decode_head(w, q, k, v, b, h)
        if i >= args.warmup:
            times.append(dt)
    per_head_bytes = 2 * w.Nk * w.d * 2
    ms = 1e3 * statistics.mean(times)
    value = per_head_bytes / (ms / 1e3) / 1e9
    sample = f"one query head per step: its decode against N_k={w.Nk} cached keys (d={w.d}) in float64"
    return {"metric": DECODE_METRIC, "value": value, "unit": "GB/s", "impl": "reference", "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{w.name}: decode B={w.B} Hq={w.Hq} Hkv={w.Hkv} Nq={w.Nq} Nk={w.Nk} d={w.d} "
                                   f"(sampled per step)"},
            "cpu_baseline": {"value": value, "unit": "GB/s", "kind": "oracle", "cores": blas_threads(),
                             "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="c3",
                    help="c2, c3, c3n, c5, c6b (bf16 fwd+bwd), c4, c6 (bf16 fwd), c1 (fp32 fwd), f3, f4 (E4M3 fwd), "
                         "f5 (E5M2 fwd), dec, dec4, dec8, dec64 (decode)")
    ap.add_argument("--shard", choices=["replicas", "heads"], default="replicas",
                    help="N>1: every rank runs the whole workload (weak scaling) or its slice of the heads (strong)")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="c3: skip timing the other workloads (c4, c5, c2, dec) after the main line")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    import synth
    world, rank, local = dist_env()
    if args.workload in synth.DECODE_WORKLOADS:
        w = synth.DECODE_WORKLOADS[args.workload]
        if args.impl == "reference":
            if rank == 0:
                print(json.dumps(run_reference_decode(args, w)), flush=True)
            return 0
        import torch
        torch.cuda.set_device(local)
        if world > 1:
            import torch.distributed as dist
            from datetime import timedelta
            dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local))
        try:
            res = run_decode(args, w, world, rank, local)
        finally:
            if world > 1:
                import torch.distributed as dist
                if dist.is_initialized():
                    dist.destroy_process_group()
        if rank == 0:
            print(json.dumps(res), flush=True)
        return 0
    w = synth.WORKLOADS[args.workload]

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, w)), flush=True)
        return 0

    import torch
    import torch.distributed as dist
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local))
    try:
        res = run_ours(args, w, world, rank, local)
    finally:
        if world > 1 and dist.is_initialized():
            dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
