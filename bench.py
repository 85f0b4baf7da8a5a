#!/usr/bin/env python
"""Benchmark of the W4A4 group-quantized GEMM hot path on B200.

One step = the whole hot path over one batch: online per-token activation quantization
(apex_quantize_act_int4) followed by the W4A4 GEMM (apex_w4a4_gemm); the weights are
packed once, offline.  Metric: effective TOPS = 2*M*N*K / step time, reported with the
roofline fraction of the dominant kernel (the GEMM).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl apex|reference]

Inputs larger than L2: every step uses the next of several copies of the packed weights
and activations, so each step reads its operands from HBM.  Under torchrun each rank runs
an independent replica (the path has no exchange step), time = max over ranks.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from group_quantized_w4a4_b200 import roofline, synth  # noqa: E402

DEFAULT_WORKLOAD = "decode_m16_n8192_k8192"
SECOND_WORKLOAD = "prefill_m4096_n8192_k8192"
INT8_PER_BF16 = 2.0   # nominal dense int8 : bf16 tensor throughput ratio on B200 (4.5 : 2.25)
INT8_SPEC_TOPS = 4500.0   # B200 dense int8 tensor throughput, public spec (context)
HBM_SPEC_GBS = 8000.0     # B200 HBM3e, public spec (context)
PREROLL_S = 0.1           # untimed replays under the clock sampler before a timed replay
PREFILL_STEPS = 100       # the tensor-bound companion line's timed steps (about 70 ms)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ distributed plumbing

def dist_init(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def job_throughput(ops_per_step: float, ms_per_step: float, world: int) -> float:
    """Whole-job TOPS: every replica ran ops_per_step per step; the step time is the
    slowest rank's."""
    return world * ops_per_step / (ms_per_step * 1e-3) / 1e12


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Polls the SM clock and the clock-event (throttle) reasons through NVML from a
    background thread while the timed region runs (read-only queries)."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, cuda_index: int):
        self.cuda_index = cuda_index
        self.samples = []
        self.stamps = []
        self.timed = None       # (t0, t1) host clock around the timed replay
        self.reasons = 0
        self.max_mhz = None
        self._stop = None
        self._thread = None
        self._err = None

    def _handle(self, nv):
        import torch
        try:
            uuid = str(torch.cuda.get_device_properties(self.cuda_index).uuid)
            return nv.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-")
                                                else uuid)
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
            idx = int(vis.split(",")[self.cuda_index]) if vis and vis.split(",")[0].isdigit() \
                else self.cuda_index
            return nv.nvmlDeviceGetHandleByIndex(idx)

    def start(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._handle(nv)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
        except Exception as e:  # no NVML: report that instead of clocks
            self._err = f"nvml unavailable: {type(e).__name__}"
            return
        self._stop = threading.Event()

        def poll():
            while not self._stop.is_set():
                try:
                    self.samples.append(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                    self.stamps.append(time.perf_counter())
                    self.reasons |= int(get_reasons(h))
                except Exception:
                    pass
                self._stop.wait(0.002)

        self._thread = threading.Thread(target=poll, daemon=True)
        self._thread.start()

    def stop(self):
        if self._thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "samples": 0,
                    "reasons": [self._err or "not sampled"]}
        self._stop.set()
        self._thread.join(timeout=2)
        names = sorted(v for k, v in self.REASONS.items() if self.reasons & k)
        in_timed = 0
        if self.timed is not None:
            t0, t1 = self.timed
            in_timed = sum(1 for t in self.stamps if t0 <= t <= t1)
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples),
                "samples_in_timed_replay": in_timed, "reasons": names,
                "source": ("NVML polled every 2 ms while the GPU ran the same CUDA graph: "
                           f"{PREROLL_S * 1e3:.0f} ms of untimed replays right before the timed "
                           "replay, then the timed replay itself")}


# ------------------------------------------------------------------ the apex arm

EXPANDED_MIN_M = 128   # from this many tokens on: one byte per activation (int8 path)
FP8_MIN_M = 1024       # from this many tokens on: the E4M3-carrier GEMM (enough 128 x 256
                       # tiles to fill the SMs at these widths)
FORM_OVERRIDE = None   # set by --form


def activation_form(M: int) -> str:
    """Operand form of the step: packed int4 (few tokens: memory-bound), the expanded int8
    activations of the int8 path (a few hundred tokens), or E4M3 codes of the same int4
    values for many tokens (compute-bound; the E4M3-carrier GEMM)."""
    if FORM_OVERRIDE:
        return FORM_OVERRIDE
    if M >= FP8_MIN_M:
        return "fp8"
    return "expanded" if M >= EXPANDED_MIN_M else "packed"


class Problem:
    """Device-resident operands for one workload, in C copies (inputs larger than L2)."""

    def __init__(self, apex, torch, g: synth.Gemm, copies: int):
        self.form = activation_form(g.M)
        self.expanded = self.form == "expanded"
        self.fp8 = self.form == "fp8"
        self.g = g
        a, w = synth.make(g)
        self.a_host = a
        dev = torch.device("cuda")
        self.x = []
        self.wp, self.sw, self.ap, self.sa = [], [], [], []
        a_d = torch.from_numpy(a).to(dev)
        w_d = torch.from_numpy(w).to(dev)
        # the weights are quantized once, offline, in the form the GEMM reads
        wp0, sw0 = apex.pack_weights_fp8(w_d, g.gw) if self.fp8 else apex.pack_weights(w_d, g.gw)
        del w_d
        for c in range(copies):
            self.x.append(a_d if c == 0 else a_d.clone())
            self.wp.append(wp0 if c == 0 else wp0.clone())
            self.sw.append(sw0 if c == 0 else sw0.clone())
            self.ap.append(torch.empty((g.M, g.K // 2 if self.form == "packed" else g.K),
                                       dtype=torch.uint8, device=dev))
            self.sa.append(torch.empty((g.M, g.K // 128), dtype=torch.float16, device=dev))
        self.y = torch.empty((g.M, g.N), dtype=torch.float16, device=dev)
        self.ws = apex.workspace(g.M, g.N, g.K, 128, g.gw)
        self.copies = copies


def copies_for(g: synth.Gemm, l2_bytes: int) -> int:
    per = g.gemm_bytes() + g.quant_bytes()
    c = 2
    while c * per < 2 * l2_bytes and c < 64:
        c += 1
    return c


def quantizer_of(apex, form):
    return {"packed": apex.apex_quantize_act_int4,
            "expanded": apex.apex_quantize_act_int4_expanded,
            "fp8": apex.apex_quantize_act_int4_fp8}[form]


def gemm_call(apex, form, g, a, sa, w, sw, y, ws, stream):
    if form == "fp8":
        apex.apex_w4a4_gemm_fp8(g.M, g.N, g.K, 128, g.gw, a, sa, w, sw, y, stream)
    else:
        gemm = apex.apex_w4a4_gemm_expanded if form == "expanded" else apex.apex_w4a4_gemm
        gemm(g.M, g.N, g.K, 128, g.gw, a, sa, w, sw, y, ws, None, stream)


def apex_quantize(apex, p: Problem, i: int, stream):
    g, c = p.g, i % p.copies
    quantizer_of(apex, p.form)(p.x[c], g.M, g.K, 128, p.ap[c], p.sa[c], stream)


def apex_gemm(apex, p: Problem, i: int, stream):
    g, c = p.g, i % p.copies
    gemm_call(apex, p.form, g, p.ap[c], p.sa[c], p.wp[c], p.sw[c], p.y, p.ws, stream)


def apex_step(apex, p: Problem, i: int, stream):
    """One step of the hot path: online activation quantize, then the W4A4 GEMM."""
    apex_quantize(apex, p, i, stream)
    apex_gemm(apex, p, i, stream)


def timed_graph(torch, fn, steps, first, world, clocks=None):
    """Capture fn(i, stream) for i = first .. first+steps-1 in one CUDA graph, replay it once
    untimed (the first replay also uploads the graph to the device, a one-time cost of a few
    microseconds per node), then replay it once more between CUDA events on the capturing
    stream (barrier + synchronize on both sides).  Kernels follow each other with no event in
    between, so each launch overlaps the tail of the previous one as it does in a real
    stream.  Returns (total ms, clock record)."""
    side = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            for i in range(steps):
                fn(first + i, side)
    torch.cuda.synchronize()
    with torch.cuda.stream(side):
        graph.replay()
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if clocks:
        # the clock record covers the GPU under this same load: untimed replays for
        # PREROLL_S first (a short timed region alone leaves NVML too few samples)
        clocks.start()
        t_end = time.perf_counter() + PREROLL_S
        with torch.cuda.stream(side):
            while time.perf_counter() < t_end:
                graph.replay()
                side.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    with torch.cuda.stream(side):
        start.record(side)
        graph.replay()
        stop.record(side)
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    barrier(world)
    clk = None
    if clocks:
        clocks.timed = (t0, t1)
        clk = clocks.stop()
        if clk.get("sm_mhz"):
            clk["ms_x_sm_mhz"] = round(start.elapsed_time(stop) * clk["sm_mhz"], 3)
    del graph
    return start.elapsed_time(stop), clk


def time_workload(apex, torch, g, steps, warmup, world, l2_bytes, clocks=None):
    """W eager warm-up steps, then three timed CUDA-graph replays of exactly K launches each:
    the K steps (quantize + GEMM; the headline), the K GEMMs alone and the K quantizer
    launches alone (per-kernel average durations for the roofline)."""
    p = Problem(apex, torch, g, copies_for(g, l2_bytes))
    stream = torch.cuda.current_stream()
    for i in range(max(warmup, p.copies)):   # every copy's quantized operands exist
        apex_step(apex, p, i, stream)
    torch.cuda.synchronize()
    if apex.apex_get_device_status() != 0:
        raise RuntimeError("device status not clean after warm-up")
    step = lambda i, s: apex_step(apex, p, i, s)
    total_ms, clk = timed_graph(torch, step, steps, warmup, world, clocks)
    gemm_ms, _ = timed_graph(torch, lambda i, s: apex_gemm(apex, p, i, s), steps, warmup, world)
    quant_ms, _ = timed_graph(torch, lambda i, s: apex_quantize(apex, p, i, s), steps, warmup,
                              world)
    if apex.apex_get_device_status() != 0:
        raise RuntimeError("device status not clean after the timed steps")
    return p, total_ms, gemm_ms / steps, clk, quant_ms / steps


def e2e_workload(apex, torch, g, steps, warmup, p: Problem):
    """Same step through the public API with host buffers, as a serving loop runs it: every
    step copies its fp16 activations in from pinned host memory, quantizes, runs the GEMM
    and copies its fp16 output back to pinned host memory, all inside the timed region.
    The copies run on their own streams, ordered by events, so step i+1's input copy and
    step i's output copy overlap the kernels (inputs rotate over the device copies, outputs
    over two device and two host buffers).  The K timed steps are one CUDA graph."""
    stream = torch.cuda.current_stream()
    copy_in, copy_out = torch.cuda.Stream(), torch.cuda.Stream()
    x_host = torch.from_numpy(p.a_host).pin_memory()
    y_dev = [p.y, torch.empty_like(p.y)]
    y_host = [torch.empty((g.M, g.N), dtype=torch.float16).pin_memory() for _ in range(2)]
    C = p.copies
    ev = lambda: torch.cuda.Event()
    in_ready, q_done = [ev() for _ in range(C)], [ev() for _ in range(C)]
    y_ready, out_done = [ev() for _ in range(2)], [ev() for _ in range(2)]
    quant = quantizer_of(apex, p.form)

    def step(j, first):
        c, b = j % C, j % 2
        with torch.cuda.stream(copy_in):
            if j - first >= C:
                copy_in.wait_event(q_done[c])          # that copy's previous reader is done
            p.x[c].copy_(x_host, non_blocking=True)
            in_ready[c].record(copy_in)
        stream.wait_event(in_ready[c])
        if j - first >= 2:
            stream.wait_event(out_done[b])             # that output's previous copy is done
        quant(p.x[c], g.M, g.K, 128, p.ap[c], p.sa[c], stream)
        q_done[c].record(stream)
        gemm_call(apex, p.form, g, p.ap[c], p.sa[c], p.wp[c], p.sw[c], y_dev[b], p.ws, stream)
        y_ready[b].record(stream)
        with torch.cuda.stream(copy_out):
            copy_out.wait_event(y_ready[b])
            y_host[b].copy_(y_dev[b], non_blocking=True)
            out_done[b].record(copy_out)

    def run(first, n, s):
        nonlocal stream
        stream = s
        copy_in.wait_stream(s)
        copy_out.wait_stream(s)
        for j in range(first, first + n):
            step(j, first)
        s.wait_stream(copy_in)
        s.wait_stream(copy_out)

    run(0, warmup, torch.cuda.current_stream())
    torch.cuda.synchronize()
    # the K timed steps, copies included, as one CUDA graph (so the host issues nothing
    # inside the timed region), replayed once untimed to upload it, then timed
    side = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            run(warmup, steps, side)
    torch.cuda.synchronize()
    with torch.cuda.stream(side):
        graph.replay()
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(side):
        start.record(side)
        graph.replay()
        stop.record(side)
    torch.cuda.synchronize()
    del graph
    ms = start.elapsed_time(stop) / steps
    return ms, x_host.numel() * 2, y_host[0].numel() * 2


def kernel_source_hash() -> str:
    """sha256 (first 16 hex) of the CUDA sources, to tell whether recorded counters still
    describe the kernel that runs."""
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "group_quantized_w4a4_b200", "csrc", "*"))):
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(name: str):
    """DRAM bytes per GEMM launch from the last ncu capture of this workload, or None when
    there is none or the kernel sources changed since it was taken."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as fh:
            rec = json.load(fh)
    except (OSError, ValueError):
        return None
    if rec.get("source_hash") != kernel_source_hash():
        return None
    return rec.get("traffic_bytes_per_launch", {}).get(name)


def measure_int8_peak(torch, reps: int = 10):
    """Dense int8 tensor throughput of this GPU, measured: torch._int_mm (cuBLASLt) on
    8192^3 int8 operands, best of `reps` launches timed with CUDA events (TOPS)."""
    n = 8192
    a = torch.randint(-8, 8, (n, n), dtype=torch.int8, device="cuda")
    b = torch.randint(-8, 8, (n, n), dtype=torch.int8, device="cuda")
    for _ in range(3):
        torch._int_mm(a, b.t())
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(reps):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        torch._int_mm(a, b.t())
        e.record()
        torch.cuda.synchronize()
        best = min(best, s.elapsed_time(e))
    del a, b
    torch.cuda.empty_cache()
    return {"tops": round(2.0 * n ** 3 / (best * 1e-3) / 1e12, 1),
            "how": f"torch._int_mm int8 {n}^3, best of {reps}, CUDA events, in this run"}


def roofline_obj(g, gemm_ms_avg, peaks, peaks_kind, traffic=None, int8_peak=None,
                 form=None):
    hbm = float(peaks["hbm_gbs"]) * 1e9
    if int8_peak is not None:
        i8 = float(int8_peak["tops"]) * 1e12
        i8_note = f"int8 measured: {int8_peak['how']}"
    else:
        i8 = float(peaks.get("bf16_tflops", 1590.0)) * 1e12 * INT8_PER_BF16
        i8_note = (f"int8 = {INT8_PER_BF16:g} x bf16_tflops of {peaks_kind} "
                   "(nominal int8:bf16 ratio)")
    nbytes = g.gemm_bytes(form or activation_form(g.M))
    t_bound, bound = roofline.bound_time_s(g.ops, nbytes, i8, hbm)
    t = gemm_ms_avg * 1e-3
    if bound == "hbm":
        achieved = nbytes / t / 1e9
        peak = float(peaks["hbm_gbs"])
        unit = "GB/s"
        note = f"hbm_gbs of {peaks_kind}"
        spec = {"peak": HBM_SPEC_GBS, "frac": round(achieved / HBM_SPEC_GBS, 4)}
    else:
        achieved = g.ops / t / 1e12
        peak = i8 / 1e12
        unit = "TOPS"
        note = i8_note
        spec = {"peak": INT8_SPEC_TOPS, "frac": round(achieved / INT8_SPEC_TOPS, 4)}
    return {"bound": "hbm" if bound == "hbm" else "tensor", "achieved": round(achieved, 2),
            "peak": round(peak, 1), "unit": unit, "frac": round(achieved / peak, 4),
            "traffic": traffic if traffic is not None else recorded_traffic(g.name),
            "peak_source": note, "spec": spec,
            "algorithmic_bytes": nbytes, "ops": g.ops,
            "kernel_ms": round(gemm_ms_avg, 5)}


def oracle_inputs(g: synth.Gemm):
    """The workload's activations and the oracle's packed weights (set up once)."""
    import oracle
    a, w = synth.make(g)
    wp, sw = oracle.quantize_pack(w, g.gw)
    return a, wp, sw


def cpu_baseline(g: synth.Gemm, budget_s: float = 20.0, repeat_small: bool = True,
                 inputs=None):
    """The oracle, as it stands, on this host's cores: quantize the activations and run the
    fp64 GEMM over a bounded sample of output rows; effective TOPS scaled to the rows."""
    import oracle
    a, wp, sw = inputs if inputs is not None else oracle_inputs(g)
    rows = np.arange(min(g.M, 4), dtype=np.int64)
    t0 = time.perf_counter()
    ap, sa = oracle.quantize_pack(a[rows], 128)
    oracle.gemm(ap, sa, wp, sw, rows.size, g.N, g.K, 128, g.gw)
    dt = time.perf_counter() - t0
    n = rows.size
    # grow the sample while it stays well inside the budget
    while n < g.M and dt * 2 < budget_s / 4:
        n = min(g.M, n * 2)
        rows = np.arange(n, dtype=np.int64)
        t0 = time.perf_counter()
        ap, sa = oracle.quantize_pack(a[rows], 128)
        oracle.gemm(ap, sa, wp, sw, n, g.N, g.K, 128, g.gw)
        dt = time.perf_counter() - t0
    # a whole small workload is repeated until about half the budget of CPU work is timed
    reps = 1
    if repeat_small and n == g.M and dt < budget_s / 2:
        reps = max(1, int(np.ceil((budget_s / 2) / max(dt, 1e-3))))
        t0 = time.perf_counter()
        for _ in range(reps):
            ap, sa = oracle.quantize_pack(a[rows], 128)
            oracle.gemm(ap, sa, wp, sw, n, g.N, g.K, 128, g.gw)
        dt = (time.perf_counter() - t0) / reps
    tops = 2.0 * n * g.N * g.K / dt / 1e12
    what = f"{n} of {g.M} token rows x all {g.N} outputs of {g.name}"
    if reps > 1:
        what = f"all of {g.name}, {reps} times"
    return {"value": round(tops, 6), "unit": "TOPS", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{what} (quantize + int64 partials + fp64 scaling), "
                      f"{dt * reps:.1f} s of CPU work timed"}


def run_apex(args, rank, world, local):
    import torch
    import group_quantized_w4a4_b200 as apex
    apex.load_library()
    torch.cuda.set_device(local)
    props = torch.cuda.get_device_properties(local)
    l2 = int(getattr(props, "L2_cache_size", 126 * 1024 * 1024))
    peaks, peaks_kind = load_peaks()
    g = synth.workloads()[args.workload]
    int8_peak = measure_int8_peak(torch)
    clocks = ClockSampler(local) if rank == 0 else None
    p, total_ms, gemm_avg, clk, quant_avg = time_workload(apex, torch, g, args.steps,
                                                          args.warmup, world, l2, clocks)
    ms_step = max_over_ranks(total_ms / args.steps, world)
    gemm_avg = max_over_ranks(gemm_avg, world)
    value = job_throughput(g.ops, ms_step, world)
    e2e_ms, hb, db = e2e_workload(apex, torch, g, max(3, args.steps), args.warmup, p)
    e2e_ms = max_over_ranks(e2e_ms, world)
    del p
    torch.cuda.empty_cache()
    extra = {}
    if not args.no_second and args.workload != SECOND_WORKLOAD:
        g2 = synth.workloads()[SECOND_WORKLOAD]
        clocks2 = ClockSampler(local) if rank == 0 else None
        p2, tot2, gm2, clk2, qm2 = time_workload(apex, torch, g2, PREFILL_STEPS,
                                                 args.warmup, world, l2, clocks2)
        gm2, qm2 = max_over_ranks(gm2, world), max_over_ranks(qm2, world)
        ms2 = max_over_ranks(tot2 / PREFILL_STEPS, world)
        extra[SECOND_WORKLOAD] = {
            "value": round(job_throughput(g2.ops, ms2, world), 2), "unit": "TOPS",
            "ms_per_step": round(ms2, 4), "steps": PREFILL_STEPS,
            "activation_form": activation_form(g2.M),
            "quantize_ms": round(qm2, 5), "gemm_ms": round(gm2, 5),
            "roofline": roofline_obj(g2, gm2, peaks, peaks_kind, int8_peak=int8_peak),
            "clocks": clk2}
        del p2
    if rank != 0:
        return None
    form = activation_form(g.M)
    line = {
        "metric": "W4A4-g128 GEMM effective TOPS (quantize + GEMM step) and % of roofline",
        "value": round(value, 2), "unit": "TOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8 MMA (int4 operands), fp32 epilogue",
        "data": "synthetic (seeded N(0,1) activations, N(0,0.02) weights, fp16)",
        "config": {"workload": g.name, "M": g.M, "N": g.N, "K": g.K, "group_a": 128,
                   "group_w": g.gw, "parallelism": f"replicas x{world}",
                   "activation_form": form,
                   "l2": f"inputs larger than L2: {p_copies(g, l2)} rotating copies"},
        "roofline": roofline_obj(g, gemm_avg, peaks, peaks_kind, int8_peak=int8_peak),
        "int8_peak_measured": int8_peak,
        "e2e": {"value": round(job_throughput(g.ops, e2e_ms, world), 3), "unit": "TOPS",
                "h2d_bytes_per_step": hb, "d2h_bytes_per_step": db,
                "ms_per_step": round(e2e_ms, 4),
                "how": ("pinned host copies in and out every step on their own streams, "
                        "overlapping the kernels; the K steps replayed as one CUDA graph")},
        "gpu_launches": 2 * args.steps,
        "launch": ("one CUDA graph of the K timed steps (eager warm-up, then one untimed "
                   "replay that uploads the graph), kernels launched as programmatic "
                   "dependents; per-kernel times from two more graphs of K launches of that "
                   "kernel alone"),
        "gemm": {"kernel_ms": round(gemm_avg, 5), "bytes": g.gemm_bytes(form)},
        "quantize": {"kernel_ms": round(quant_avg, 5), "bytes": g.quant_bytes(form),
                     "GB/s": round(g.quant_bytes(form) / (quant_avg * 1e-3) / 1e9, 1)},
        "clocks": clk,
        "impl": "apex",
    }
    if extra:
        line["also"] = extra
    if world == 1 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline(g)
    return line


def run_sweep(args, rank, world, local):
    """One JSON line per secondary workload: the mixed-granularity sweep (M x weight group)
    and the MLP pair, each timed like the headline (step, GEMM alone, quantizer alone)."""
    import torch
    import group_quantized_w4a4_b200 as apex
    apex.load_library()
    torch.cuda.set_device(local)
    props = torch.cuda.get_device_properties(local)
    l2 = int(getattr(props, "L2_cache_size", 126 * 1024 * 1024))
    peaks, peaks_kind = load_peaks()
    names = [n for n in synth.workloads() if n.startswith("sweep_") or n.startswith("mlp_")]
    steps = max(3, args.steps // 4)
    int8_peak = measure_int8_peak(torch)
    lines = []
    for name in names:
        g = synth.workloads()[name]
        p, tot, gm, _, qm = time_workload(apex, torch, g, steps, args.warmup, world, l2)
        del p
        torch.cuda.empty_cache()
        ms = max_over_ranks(tot / steps, world)
        gm, qm = max_over_ranks(gm, world), max_over_ranks(qm, world)
        lines.append({
            "sweep": name, "M": g.M, "N": g.N, "K": g.K, "group_a": 128, "group_w": g.gw,
            "steps": steps, "activation_form": activation_form(g.M),
            "step_ms": round(ms, 5), "gemm_ms": round(gm, 5), "quantize_ms": round(qm, 5),
            "step_TOPS": round(job_throughput(g.ops, ms, world), 2),
            "gemm_TOPS": round(g.ops / (gm * 1e-3) / 1e12, 2),
            "gemm_GBs": round(g.gemm_bytes(activation_form(g.M)) / (gm * 1e-3) / 1e9, 1),
            "roofline": roofline_obj(g, gm, peaks, peaks_kind, int8_peak=int8_peak)})
    for m in (2048, 16):
        line = chain_line(apex, torch, m, steps, args.warmup, world)
        lines.append(line)
    lines.append(fp8_chain_line(apex, torch, 2048, steps, args.warmup, world))
    lines.append(dual_line(apex, torch, synth.workloads()[SECOND_WORKLOAD], steps, args.warmup,
                           world, l2, peaks, peaks_kind, int8_peak))
    return lines if rank == 0 else None


def fp8_chain_line(apex, torch, M, steps, warmup, world):
    """The MLP pair (8192 -> 28672 -> 8192) chained on the E4M3 path, timed as one step two
    ways: the up layer writing the down layer's E4M3-coded activations in its epilogue
    (apex_w4a4_gemm_fp8_quant), and unfused (fp16 output, then the E4M3 quantizer)."""
    up, down = synth.workloads()["mlp_up_m2048_n28672_k8192"], \
        synth.workloads()["mlp_down_m2048_n8192_k28672"]
    K, H, N = up.K, up.N, down.N
    dev = torch.device("cuda")
    x = torch.from_numpy(synth.activations(M, K, "student_t", 7)).to(dev)
    w1 = torch.from_numpy(synth.weights(H, K, 8)).to(dev)
    w1c, w1s = apex.pack_weights_fp8(w1, 128)
    del w1
    w2 = torch.from_numpy(synth.weights(N, H, 9)).to(dev)
    w2c, w2s = apex.pack_weights_fp8(w2, 128)
    del w2
    xa = torch.empty((M, K), dtype=torch.uint8, device=dev)
    xs = torch.empty((M, K // 128), dtype=torch.float16, device=dev)
    ha = torch.empty((M, H), dtype=torch.uint8, device=dev)
    hs = torch.empty((M, H // 128), dtype=torch.float16, device=dev)
    hy = torch.empty((M, H), dtype=torch.float16, device=dev)
    y = torch.empty((M, N), dtype=torch.float16, device=dev)

    def fused(i, s):
        apex.apex_quantize_act_int4_fp8(x, M, K, 128, xa, xs, s)
        apex.apex_w4a4_gemm_fp8_quant(M, H, K, 128, 128, xa, xs, w1c, w1s, None, ha, hs, s)
        apex.apex_w4a4_gemm_fp8(M, N, H, 128, 128, ha, hs, w2c, w2s, y, s)

    def unfused(i, s):
        apex.apex_quantize_act_int4_fp8(x, M, K, 128, xa, xs, s)
        apex.apex_w4a4_gemm_fp8(M, H, K, 128, 128, xa, xs, w1c, w1s, hy, s)
        apex.apex_quantize_act_int4_fp8(hy, M, H, 128, ha, hs, s)
        apex.apex_w4a4_gemm_fp8(M, N, H, 128, 128, ha, hs, w2c, w2s, y, s)

    stream = torch.cuda.current_stream()
    for i in range(warmup):
        fused(i, stream)
        unfused(i, stream)
    torch.cuda.synchronize()
    if apex.apex_get_device_status() != 0:
        raise RuntimeError("device status not clean after the chain warm-up")
    f_ms, _ = timed_graph(torch, fused, steps, warmup, world)
    u_ms, _ = timed_graph(torch, unfused, steps, warmup, world)
    f_ms = max_over_ranks(f_ms / steps, world)
    u_ms = max_over_ranks(u_ms / steps, world)
    ops = 2.0 * M * K * H + 2.0 * M * H * N
    return {"sweep": f"mlp_chain_fp8_m{M}", "M": M, "K": K, "hidden": H, "N": N,
            "activation_form": "fp8", "steps": steps,
            "fused_step_ms": round(f_ms, 5), "unfused_step_ms": round(u_ms, 5),
            "fused_TOPS": round(job_throughput(ops, f_ms, world), 2),
            "unfused_TOPS": round(job_throughput(ops, u_ms, world), 2),
            "what": ("x -> quantize -> up (8192 -> 28672) -> down (28672 -> 8192) on the E4M3 "
                     "path; fused: the up layer writes the down layer's E4M3 codes and scales "
                     "in its epilogue; unfused: fp16 output, then the quantizer")}


def dual_line(apex, torch, g, steps, warmup, world, l2, peaks, peaks_kind, int8_peak):
    """The outlier dual path on a workload with persistent outlier channels (the prefill
    workload: 1% of K, x20, the same for every token): the step is the dual quantizer (the
    outlier channels to fp16, the rest to E4M3 codes) and the dual GEMM (the 4-bit groups plus
    the 16-bit outlier K-steps), timed as the plain step is."""
    dev = torch.device("cuda")
    a, w = synth.make(g)
    ch = synth.outlier_channels(g.K, g.seed * 16 + 2)
    C = len(ch)
    Cp = -(-C // 64) * 64
    ch_d = torch.from_numpy(ch.astype(np.int32)).to(dev)
    w_d = torch.from_numpy(w).to(dev)
    w_out = torch.empty((g.N, Cp), dtype=torch.float16, device=dev)
    apex.apex_gather_weight_columns(w_d, g.N, g.K, ch_d, C, w_out, Cp)
    wc, sw = apex.pack_weights_fp8(w_d, g.gw)
    del w_d
    copies = copies_for(g, l2)
    xs = [torch.from_numpy(a).to(dev) for _ in range(copies)]
    qs = [torch.empty((g.M, g.K), dtype=torch.uint8, device=dev) for _ in range(copies)]
    ss = [torch.empty((g.M, g.K // 128), dtype=torch.float16, device=dev) for _ in range(copies)]
    xo = [torch.empty((g.M, Cp), dtype=torch.float16, device=dev) for _ in range(copies)]
    y = torch.empty((g.M, g.N), dtype=torch.float16, device=dev)

    def quant(i, s):
        c = i % copies
        apex.apex_quantize_act_int4_dual(xs[c], g.M, g.K, 128, ch_d, C, apex.APEX_FORM_FP8,
                                         qs[c], ss[c], xo[c], Cp, s)

    def gemm(i, s):
        c = i % copies
        apex.apex_w4a4_gemm_fp8_dual(g.M, g.N, g.K, 128, g.gw, qs[c], ss[c], wc, sw, xo[c],
                                     w_out, Cp, y, s)

    def step(i, s):
        quant(i, s)
        gemm(i, s)

    stream = torch.cuda.current_stream()
    for i in range(max(warmup, copies)):
        step(i, stream)
    torch.cuda.synchronize()
    if apex.apex_get_device_status() != 0:
        raise RuntimeError("device status not clean after the dual-path warm-up")
    tot, _ = timed_graph(torch, step, steps, warmup, world)
    gm, _ = timed_graph(torch, gemm, steps, warmup, world)
    qm, _ = timed_graph(torch, quant, steps, warmup, world)
    ms, gm, qm = (max_over_ranks(v / steps, world) for v in (tot, gm, qm))
    return {"sweep": f"{g.name}_outlier_dual", "M": g.M, "N": g.N, "K": g.K,
            "outlier_channels": C, "Cp": Cp, "steps": steps, "activation_form": "fp8",
            "step_ms": round(ms, 5), "gemm_ms": round(gm, 5), "quantize_ms": round(qm, 5),
            "step_TOPS": round(job_throughput(g.ops, ms, world), 2),
            "roofline": roofline_obj(g, gm, peaks, peaks_kind, int8_peak=int8_peak,
                                     form="fp8"),
            "what": ("outlier channels in fp16 through extra kind::f16 K-steps of the same "
                     "GEMM, the rest W4A4-g128; ops counted as the plain GEMM's 2*M*N*K")}


def chain_line(apex, torch, M, steps, warmup, world):
    """Two chained W4A4 layers (the MLP pair's shapes: 8192 -> 28672 -> 8192), timed as one
    step two ways: with the first layer's output quantized in its epilogue for the second
    (apex_w4a4_gemm_quant), and unfused (fp16 output, then the activation quantizer)."""
    up, down = synth.workloads()["mlp_up_m2048_n28672_k8192"], \
        synth.workloads()["mlp_down_m2048_n8192_k28672"]
    K, H, N = up.K, up.N, down.N
    exp = M >= EXPANDED_MIN_M   # the quantized-output epilogue belongs to the int8 path
    dev = torch.device("cuda")
    x = torch.from_numpy(synth.activations(M, K, "student_t", 7)).to(dev)
    w1 = torch.from_numpy(synth.weights(H, K, 8)).to(dev)
    w1p, w1s = apex.pack_weights(w1, 128)
    del w1
    w2 = torch.from_numpy(synth.weights(N, H, 9)).to(dev)
    w2p, w2s = apex.pack_weights(w2, 128)
    del w2
    xa = torch.empty((M, K if exp else K // 2), dtype=torch.uint8, device=dev)
    xs = torch.empty((M, K // 128), dtype=torch.float16, device=dev)
    ha = torch.empty((M, H if exp else H // 2), dtype=torch.uint8, device=dev)
    hs = torch.empty((M, H // 128), dtype=torch.float16, device=dev)
    hy = torch.empty((M, H), dtype=torch.float16, device=dev)
    y = torch.empty((M, N), dtype=torch.float16, device=dev)
    ws1, ws2 = apex.workspace(M, H, K), apex.workspace(M, N, H)
    quant = apex.apex_quantize_act_int4_expanded if exp else apex.apex_quantize_act_int4
    gemm = apex.apex_w4a4_gemm_expanded if exp else apex.apex_w4a4_gemm
    gemm_q = apex.apex_w4a4_gemm_expanded_quant if exp else apex.apex_w4a4_gemm_quant

    def fused(i, s):
        quant(x, M, K, 128, xa, xs, s)
        gemm_q(M, H, K, 128, 128, xa, xs, w1p, w1s, None, ha, hs, exp, ws1, None, s)
        gemm(M, N, H, 128, 128, ha, hs, w2p, w2s, y, ws2, None, s)

    def unfused(i, s):
        quant(x, M, K, 128, xa, xs, s)
        gemm(M, H, K, 128, 128, xa, xs, w1p, w1s, hy, ws1, None, s)
        quant(hy, M, H, 128, ha, hs, s)
        gemm(M, N, H, 128, 128, ha, hs, w2p, w2s, y, ws2, None, s)

    stream = torch.cuda.current_stream()
    for i in range(warmup):
        fused(i, stream)
        unfused(i, stream)
    torch.cuda.synchronize()
    if apex.apex_get_device_status() != 0:
        raise RuntimeError("device status not clean after the chain warm-up")
    f_ms, _ = timed_graph(torch, fused, steps, warmup, world)
    u_ms, _ = timed_graph(torch, unfused, steps, warmup, world)
    f_ms = max_over_ranks(f_ms / steps, world)
    u_ms = max_over_ranks(u_ms / steps, world)
    ops = 2.0 * M * K * H + 2.0 * M * H * N
    return {"sweep": f"mlp_chain_m{M}", "M": M, "K": K, "hidden": H, "N": N,
            "activation_form": "expanded" if exp else "packed", "steps": steps,
            "fused_step_ms": round(f_ms, 5), "unfused_step_ms": round(u_ms, 5),
            "fused_TOPS": round(job_throughput(ops, f_ms, world), 2),
            "unfused_TOPS": round(job_throughput(ops, u_ms, world), 2),
            "what": ("x -> quantize -> up (8192 -> 28672) -> down (28672 -> 8192); fused: the "
                     "up layer writes the down layer's int4 operand in its epilogue; unfused: "
                     "fp16 output, then the activation quantizer")}


def p_copies(g, l2):
    return copies_for(g, l2)


def run_reference(args, rank, world):
    """The oracle, as it stands, on the host cores, for the same workload and metric."""
    if rank != 0:
        return None
    g = synth.workloads()[args.workload]
    # each step a bounded sample, sized so that the whole run stays near two minutes
    per_step = max(0.02, 120.0 / (args.steps + args.warmup))
    inputs = oracle_inputs(g)
    vals = []
    for _ in range(args.warmup):
        cpu_baseline(g, budget_s=per_step, repeat_small=False, inputs=inputs)
    for _ in range(args.steps):
        vals.append(cpu_baseline(g, budget_s=per_step, repeat_small=False, inputs=inputs))
    v = statistics.median([x["value"] for x in vals])
    cb = dict(vals[-1])
    cb["value"] = v
    return {"metric": "W4A4-g128 GEMM effective TOPS (quantize + GEMM step) and % of roofline",
            "value": v, "unit": "TOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup,
            # one whole step of the workload at the sampled rate
            "ms_per_step": round(g.ops / (v * 1e12) * 1e3, 3) if v > 0 else None,
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int64 partials, fp64 scaling", "data": "synthetic",
            "config": {"workload": g.name, "M": g.M, "N": g.N, "K": g.K, "group_a": 128,
                       "group_w": g.gw},
            "impl": "reference", "cpu_baseline": cb,
            "e2e": {"value": v, "unit": "TOPS", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.workloads()))
    ap.add_argument("--impl", default="apex", choices=["apex", "reference"])
    ap.add_argument("--no-cpu", action="store_true", help="skip the cpu_baseline leg")
    ap.add_argument("--no-second", action="store_true", help="skip the M=4096 companion line")
    ap.add_argument("--sweep", action="store_true",
                    help="instead of the headline line, one line per sweep / MLP workload")
    ap.add_argument("--form", choices=["packed", "expanded", "fp8"], default=None,
                    help="operand form of every step (default: by the number of tokens)")
    args = ap.parse_args()
    global FORM_OVERRIDE
    FORM_OVERRIDE = args.form
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank, world, local = dist_init(args.gpus)
    try:
        if args.sweep:
            for line in run_sweep(args, rank, world, local) or []:
                print(json.dumps(line), flush=True)
        else:
            if args.impl == "reference":
                line = run_reference(args, rank, world)
            else:
                line = run_apex(args, rank, world, local)
            if line is not None:
                print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
