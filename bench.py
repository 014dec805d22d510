#!/usr/bin/env python
"""Throughput of the chunked GDN scan on B200: head-tokens/s and latent
frames/s on the 1280x704 streaming chunk, with the roofline fraction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

A step is one library call on one streaming chunk: B1 x H20 x T2640 tokens
(3 latent frames of 40x22), d_k = d_v = 112, bf16 q/k/v/out, fp32 g, beta and
carried state -- the causal scan with the previous chunk's state.  Inputs are
resident in HBM before timing starts and rotate over enough buffer sets that
their total exceeds L2 (so every step reads from HBM).  Steps are timed with
CUDA events on the launching stream, K steps between a barrier + synchronize
on both sides, max over ranks.  With N > 1 (torchrun) every rank scans its own
chunk stream: the work partitions over independent chunks with no exchange,
so scaling is weak and no collective sits on the data path.

``--impl reference`` times the fp64 CPU oracle (token recurrence) on the same
workload on this host's cores instead (rank 0 only).

Rank 0 prints one JSON line.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "GDN head-tokens/s and latent frames/s at 2640-tok chunk; % of B200 roofline"
UNIT = "head-tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
N_SETS = 8                      # rotating input sets (8 x 49.7 MB > 126 MB L2)
KERNEL_SOURCES = {
    "gdn_scan_serial_kernel": "gated_deltanet_linear_chunked_b200/csrc/scan_serial.cu",
    "gdn_prep_kernel": "gated_deltanet_linear_chunked_b200/csrc/chunk_tc.cu",
    "gdn_recur_kernel": "gated_deltanet_linear_chunked_b200/csrc/chunk_tc.cu",
    "gdn_output_kernel": "gated_deltanet_linear_chunked_b200/csrc/chunk_tc.cu",
}


def parse():
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=400)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["native", "reference"], default="native")
    p.add_argument("--mode", choices=["fwd", "bidir"], default="fwd",
                   help="causal chunk (the headline workload) or the bidirectional chunk")
    p.add_argument("--no-graph", action="store_true", help="time direct calls instead of CUDA-graph replays")
    p.add_argument("--cpu-seconds", type=float, default=10.0, help="budget of the oracle CPU baseline")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-extras", action="store_true", help="skip every side figure")
    p.add_argument("--extras", default="all",
                   help="comma list of side figures: side (the other mode, the 32x15 stack, "
                        "gate logits), long (long streams), backward, sink_window; or all")
    return p.parse_args()


def load_peaks():
    """The roofline denominators and where they came from.  Each of the three
    peaks is taken from MEASURED_PEAKS.json when the file holds it as a
    number, else from FALLBACK_PEAKS; an absent or unreadable file counts as
    holding none.  The second value names the source for the peak_source
    fields: "measured", "fallback", or "measured, with fallback for <keys>"."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        d = {}
    if not isinstance(d, dict):
        d = {}
    peaks, missing = {}, []
    for key, fallback in FALLBACK_PEAKS.items():
        v = d.get(key)
        try:
            v = float(v)
        except (TypeError, ValueError):
            v = None
        if v is None or not v > 0:
            peaks[key] = fallback
            missing.append(key)
        else:
            peaks[key] = v
    if not missing:
        return peaks, "measured"
    if len(missing) == len(FALLBACK_PEAKS):
        return peaks, "fallback"
    return peaks, "measured, with fallback for " + " and ".join(missing)


def gate_keys(w):
    """Input names of the gates: g and beta, or the gate layer's logits for
    the fused-prologue workloads."""
    return ("g_logit", "beta_logit") if w.gate[0] == "logit_normal" else ("g", "beta")


def algorithmic_bytes(w) -> int:
    """q, k, v, out (dtype) + g, beta (fp32; gate logits in the dtype) per
    token-head, plus the fp32 state read and written once per (b, h)."""
    es = 2 if w.dtype == "bf16" else 4
    per_tok = (2 * w.Dk + 2 * w.Dv) * es + (2 * es if w.gate[0] == "logit_normal" else 8)
    return w.head_tokens * per_tok + 2 * w.B * w.H * w.Dk * w.Dv * 4


def algorithmic_flops(w, bidir=False) -> int:
    """Chunked-form work per token-head: 6 d^2 + 8 C d (doubled for bidir)."""
    d = w.Dk
    f = w.head_tokens * (6 * d * d + 8 * w.chunk * d)
    return 2 * f if bidir else f


def kernel_algorithmic_bytes(name, w) -> int:
    """Each kernel's share of the path's algorithmic bytes: stage A reads k, v,
    g, beta; stage B reads and writes the state; stage C reads q (and g) and
    writes out.  The token-serial kernel does all of it.  The shares sum to
    the path's bytes (q, k, v, out, g, beta + state)."""
    es = 2 if w.dtype == "bf16" else 4
    state = 2 * w.B * w.H * w.Dk * w.Dv * 4
    if name == "gdn_prep_kernel":
        return w.head_tokens * ((w.Dk + w.Dv) * es + 8)
    if name == "gdn_recur_kernel":
        return state
    if name == "gdn_output_kernel":
        return w.head_tokens * ((w.Dk + w.Dv) * es)
    return algorithmic_bytes(w)


def recorded_traffic(kernel):
    """DRAM bytes per launch of `kernel` on this workload from the committed
    ncu summary (profiles/dram_traffic.txt), if the summary was taken on the
    kernel's current source; else None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None
    src_path = KERNEL_SOURCES.get(kernel)
    if src_path is None:
        return None
    try:
        digest = hashlib.sha256(open(os.path.join(ROOT, src_path), "rb").read()).hexdigest()
    except OSError:
        return None
    for line in lines:
        if line.startswith("#") or not line.strip():
            continue
        parts = line.split()
        # kernel  source_sha256  dram_bytes_per_launch
        if len(parts) >= 3 and parts[0] == kernel and parts[1] == digest:
            try:
                return int(float(parts[2]))
            except ValueError:
                return None
    return None


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML every ~5 ms (a
    timed region of 20-400 graph replays lasts only tens of milliseconds)."""

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._thr = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    _REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def _sample(self):
        nv = self.nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        mask = get(self.h)
        for bit, name in self._REASONS.items():
            if mask & bit:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                pass
            self._stop.wait(0.005)

    def __enter__(self):
        if self.nv is not None:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thr is not None:
            self._thr.join()
            try:
                self._sample()
            except Exception:
                pass

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


def cpu_baseline(w, budget_s: float):
    """The fp64 oracle (as it stands) on this host's cores, on the full
    streaming chunk, repeated until `budget_s` seconds have been spent."""
    import oracle
    from gated_deltanet_linear_chunked_b200 import workloads as wl
    x = wl.make_inputs(w)
    fn = oracle.oracle_bidir if w.mode == "bidir" else oracle.oracle_fwd
    cores = min(oracle.online_cores(), w.B * w.H)   # the pool never exceeds one thread per head
    reps, t0 = 0, time.perf_counter()
    while True:
        fn(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state_in"], nthreads=cores)
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s or reps >= 1000:
            break
    # the same recurrence on one core, over one head of the chunk, for about
    # a tenth of the budget
    from gated_deltanet_linear_chunked_b200.workloads import slice_head
    one = slice_head(x, 0, 0)
    reps1, t1 = 0, time.perf_counter()
    while True:
        fn(one["q"], one["k"], one["v"], one["g"], one["beta"], one["state_in"], nthreads=1)
        reps1 += 1
        el1 = time.perf_counter() - t1
        if el1 >= budget_s / 10 or reps1 >= 1000:
            break
    return {"value": w.head_tokens * reps / el, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"full {w.name} chunk (B{w.B} H{w.H} T{w.T} d{w.Dk}, fp64 token recurrence), "
                      f"{reps} repetitions in {el:.1f} s",
            "value_1core": w.T * reps1 / el1,
            "sample_1core": f"one head of the chunk on one thread, {reps1} repetitions in {el1:.1f} s"}


# ---- multi-rank plumbing (one process per GPU; no data-path collective)
def rank_workload(w, rank: int):
    """The chunk stream rank `rank` scans: the same shapes and distributions
    as `w`, its own seed, so ranks process independent streams."""
    from gated_deltanet_linear_chunked_b200 import workloads as wl
    return wl.stream_chunk(w.mode, seed=w.seed + 7919 * rank)


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest of every rank's `x` (device times are reported as the
    slowest rank's)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, steps: int, head_tokens: int, ms: float) -> float:
    """Whole-job head-tokens/s: every rank's units over the slowest rank's time."""
    return world * steps * head_tokens / (ms / 1000.0)


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    from gated_deltanet_linear_chunked_b200 import workloads as wl
    x = wl.make_inputs(w)
    fn = oracle.oracle_bidir if w.mode == "bidir" else oracle.oracle_fwd
    cores = min(oracle.online_cores(), w.B * w.H)   # the pool never exceeds one thread per head
    # size one step so the whole run stays within a few minutes
    t0 = time.perf_counter()
    fn(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state_in"], nthreads=cores)
    one = time.perf_counter() - t0
    heads = w.H
    budget_per_step = 120.0 / max(1, args.steps + args.warmup)
    if one > budget_per_step:
        heads = max(1, int(w.H * budget_per_step / one))
    xs = {n: x[n][:, :, :heads].copy() for n in ("q", "k", "v", "g", "beta")}
    s_in = None if x["state_in"] is None else x["state_in"][:, :heads].copy()
    for _ in range(args.warmup):
        fn(xs["q"], xs["k"], xs["v"], xs["g"], xs["beta"], s_in, nthreads=cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        fn(xs["q"], xs["k"], xs["v"], xs["g"], xs["beta"], s_in, nthreads=cores)
    el = time.perf_counter() - t0
    ht = w.B * heads * w.T * args.steps
    value = ht / el
    sample = (f"{heads} of {w.H} heads of the {w.name} chunk (T{w.T}, d{w.Dk}) per step, "
              f"fp64 token recurrence")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000 * el / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": heads, "T": w.T, "Dk": w.Dk, "Dv": w.Dv,
                   "mode": w.mode, "latent_frames_per_chunk": w.T / 880},
        "latent_frames_per_s": value / (w.B * heads * 880),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def nvtx(name):
    """NVTX range around a bench phase (visible in a profiler's timeline)."""
    import contextlib
    import torch
    try:
        return torch.cuda.nvtx.range(name)
    except Exception:
        return contextlib.nullcontext()


def make_sets(w, xh, dev, n):
    """`n` device copies of one chunk's inputs, each with its own out and
    state_out, so consecutive steps read different buffers."""
    import torch
    dt = torch.bfloat16
    gk = gate_keys(w)
    base = {k: torch.from_numpy(xh[k]).to(dev) for k in ("q", "k", "v", *gk)}
    for k in ("q", "k", "v") + (gk if gk[0] == "g_logit" else ()):
        base[k] = base[k].to(dt)
    base["state_in"] = torch.from_numpy(xh["state_in"]).to(dev)
    sets = []
    for _ in range(n):
        s = {k: t.clone() for k, t in base.items()}
        s["out"] = torch.empty((w.B, w.T, w.H, w.Dv), dtype=dt, device=dev)
        s["state_out"] = torch.empty_like(s["state_in"])
        sets.append(s)
    return base, sets


class Stepper:
    """One library call per step over rotating input sets, as direct calls or
    as replays of one captured CUDA graph per set.  A direct call on the
    stream comes first, so the library's per-stream scratch exists before any
    capture and the graphs hold kernel nodes only (no memory nodes)."""

    def __init__(self, fn, sets, stream, chunk, use_graph, gates=("g", "beta")):
        import torch
        self.fn, self.sets, self.stream, self.chunk, self.gates = fn, sets, stream, chunk, gates
        self.graphs = []
        with torch.cuda.stream(stream):
            self.call(0)
        torch.cuda.synchronize()
        if use_graph:
            for i in range(len(sets)):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    self.call(i)
                self.graphs.append(g)
            torch.cuda.synchronize()

    def call(self, i):
        s = self.sets[i % len(self.sets)]
        self.fn(s["q"], s["k"], s["v"], s[self.gates[0]], s[self.gates[1]], s["state_in"],
                state_out=s["state_out"], out=s["out"], chunk=self.chunk, stream=self.stream)

    def run(self, n, offset=0):
        import torch
        with torch.cuda.stream(self.stream):
            for i in range(n):
                if self.graphs:
                    self.graphs[(i + offset) % len(self.graphs)].replay()
                else:
                    self.call(i + offset)

    def warm(self, n):
        """At least `n` steps, and every graph replayed at least once."""
        self.run(max(n, len(self.sets)))

    def release(self):
        self.graphs.clear()


def kernel_times(lib, step_fn, n, launches_per_step):
    """Per-kernel CUDA-event times (the library records events on the
    launching stream around each launch) over `n` direct calls."""
    import ctypes
    from gated_deltanet_linear_chunked_b200 import _lib
    _lib.check(lib.gdn_profile_begin(int(n * max(1, launches_per_step) + 8)), "gdn_profile_begin")
    for i in range(n):
        step_fn(i)
    kms = (ctypes.c_float * 11)()
    kn = (ctypes.c_int * 11)()
    _lib.check(lib.gdn_profile_end(ctypes.addressof(kms), ctypes.addressof(kn), 11), "gdn_profile_end")
    kernels = {}
    for i in range(11):
        if kn[i]:
            kernels[lib.gdn_kernel_name(i).decode()] = {"launches": kn[i], "ms_per_launch": kms[i] / kn[i]}
    tot = sum(v["ms_per_launch"] for v in kernels.values())
    for v in kernels.values():
        v["share"] = v["ms_per_launch"] / tot if tot else None
    return kernels


def device_stream_inputs(w, dev, seed):
    """Inputs of a long stream drawn on the device (torch generator, seeded)
    with the workload's distributions -- q, k ~ N(0,1) rows L2-normalised, v
    ~ N(0,1), g ~ U[lo, hi], beta constant, state_in ~ N(0, 0.02^2) -- so a
    multi-GB stream needs no host round trip.  Timing only."""
    import torch
    gen = torch.Generator(device=dev).manual_seed(seed)
    bf = torch.bfloat16

    def rows(D):
        x = torch.randn((w.B, w.T, w.H, D), generator=gen, device=dev)
        return x / x.norm(dim=-1, keepdim=True)
    x = {"q": rows(w.Dk).to(bf), "k": rows(w.Dk).to(bf),
         "v": torch.randn((w.B, w.T, w.H, w.Dv), generator=gen, device=dev).to(bf)}
    lo, hi = w.gate[1], w.gate[2]
    x["g"] = lo + (hi - lo) * torch.rand((w.B, w.T, w.H), generator=gen, device=dev)
    x["beta"] = torch.full((w.B, w.T, w.H), float(w.beta[1]), device=dev)
    x["state_in"] = w.state[1] * torch.randn((w.B, w.H, w.Dk, w.Dv), generator=gen, device=dev)
    x["out"] = torch.empty((w.B, w.T, w.H, w.Dv), dtype=bf, device=dev)
    x["state_out"] = torch.empty_like(x["state_in"])
    return x


def time_calls(fn, x, stream, barrier, reps=3, warm=2):
    """Mean ms of `reps` direct calls after `warm` (CUDA events)."""
    import torch
    call = lambda: fn(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state_in"],  # noqa: E731
                      state_out=x["state_out"], out=x["out"], stream=stream)
    with torch.cuda.stream(stream):
        for _ in range(warm):
            call()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(reps):
            call()
    e1.record(stream)
    barrier()
    return e0.elapsed_time(e1) / reps


def long_stream_figures(gdn, lib, w, stream, dev, peaks, peak_kind, barrier):
    """The stress workload's longest case (B4 H16 d128 T65536, fast decay,
    beta 0.99) against its HBM roofline, and one head of it (B1 H1) with and
    without time segments: 1024 dependent chunk steps against the
    segmented scan's 2 ceil(1024 / G) + G."""
    import dataclasses
    from gated_deltanet_linear_chunked_b200 import workloads as wl
    res = {}
    ws = [c for c in wl.stress_cases() if c.T == 65536 and c.Dk == 128][-1]
    x = device_stream_inputs(ws, dev, 5)
    ms = time_calls(gdn.chunk_fwd, x, stream, barrier)
    t_hbm, t_tc = roofline_times(ws, False, peaks)
    res["stress_B4_H16_d128_T65536"] = {
        "workload": ws.name, "ms_per_call": ms, "head_tokens_per_s": ws.head_tokens / (ms / 1000.0),
        "roofline": {"bound": "hbm", "roofline_us": 1e6 * max(t_hbm, t_tc),
                     "algorithmic_bytes": algorithmic_bytes(ws),
                     "achieved_gbs": algorithmic_bytes(ws) / (ms / 1000.0) / 1e9,
                     "frac": (algorithmic_bytes(ws) / (ms / 1000.0) / 1e9) / peaks["hbm_gbs"],
                     "peak_source": f"{peak_kind} hbm_gbs"}}
    del x
    import torch
    torch.cuda.empty_cache()
    w1 = dataclasses.replace(ws, B=1, H=1, name="long_stream_B1_H1_d128_T65536")
    x = device_stream_inputs(w1, dev, 6)
    nC = (w1.T + 63) // 64
    old = lib.gdn_set_time_segments(1)
    try:
        ms_serial = time_calls(gdn.chunk_fwd, x, stream, barrier)
    finally:
        lib.gdn_set_time_segments(old)
    ms_seg = time_calls(gdn.chunk_fwd, x, stream, barrier)

    def seg_call(i):
        with torch.cuda.stream(stream):
            gdn.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state_in"],
                          state_out=x["state_out"], out=x["out"], stream=stream)
    split = kernel_times(lib, seg_call, 2, 5)
    G = int(round(nC ** 0.5))
    res["long_stream_time_segments"] = {
        "workload": w1.name, "chunks": nC,
        "unsegmented": {"ms_per_call": ms_serial, "serial_chunk_steps": nC},
        "segmented": {"ms_per_call": ms_seg, "segments_automatic": "about sqrt(chunks)",
                      "kernels": split,
                      "serial_chunk_steps_if_G_is_sqrt": 2 * ((nC + G - 1) // G) + G},
        "speedup": ms_serial / ms_seg}
    return res


def backward_figure(gdn, lib, base, w, stream, peaks, peak_kind, barrier):
    """The gradients of the bidirectional streaming chunk (the pages' short
    bidirectional training) with respect to q, k, v, g, beta and the carried
    state, given d_out and d_state_out.  Algorithmic bytes per token-head:
    q, k, v, d_out in and dq, dk, dv out (bf16), g, beta in and dg, dbeta out
    (fp32); plus three fp32 states per (b, h)."""
    import torch
    d_out = torch.randn_like(base["q"][..., :w.Dv].float()).to(base["q"].dtype)
    d_S = torch.randn_like(base["state_in"])

    def call():
        return gdn.chunk_bidir_backward(base["q"], base["k"], base["v"], base["g"], base["beta"],
                                        base["state_in"], d_out, d_S, stream=stream)
    with torch.cuda.stream(stream):
        for _ in range(2):
            call()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 3
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(reps):
            call()
    e1.record(stream)
    barrier()
    ms = e0.elapsed_time(e1) / reps

    def direct(i):
        with torch.cuda.stream(stream):
            call()
    split = kernel_times(lib, direct, 2, 2)
    per_tok = (4 * w.Dk + 3 * w.Dv) * 2 + 16
    nbytes = w.head_tokens * per_tok + 3 * w.B * w.H * w.Dk * w.Dv * 4
    gbs = nbytes / (ms / 1000.0) / 1e9
    # the tensor pipe binds first: the forward's products recomputed, then
    # twice them for the gradients
    flops = 3 * algorithmic_flops(w, True)
    tflops = flops / (ms / 1000.0) / 1e12
    tpeak = peaks["bf16_tflops_sustained"]
    return {"workload": "stream_chunk_bidir (gradients)", "ms_per_call": ms,
            "head_tokens_per_s": w.head_tokens / (ms / 1000.0), "kernels": split,
            "roofline": {"bound": "hbm", "algorithmic_bytes": nbytes, "achieved_gbs": gbs,
                         "peak": peaks["hbm_gbs"], "frac": gbs / peaks["hbm_gbs"],
                         "roofline_us": 1e6 * nbytes / (peaks["hbm_gbs"] * 1e9),
                         "peak_source": f"{peak_kind} hbm_gbs",
                         "tensor": {"algorithmic_flops": flops, "achieved_tflops": tflops,
                                    "peak": tpeak, "frac": tflops / tpeak,
                                    "roofline_us": 1e6 * flops / (tpeak * 1e12),
                                    "peak_source": f"{peak_kind} bf16_tflops_sustained"}}}


def sink_window_figure(gdn, lib, stream, dev, peaks, peak_kind, barrier):
    """The softmax blocks' attention on the streaming chunk: B1 H20 D112
    Tc2640, one sink chunk and a window of two, at a steady-state chunk
    (index 5: the sink, chunk 4 and its own, 7920 keys per query).  Inputs
    and caches rotate over three sets (each about 94 MB of reads and writes,
    together more than L2).  Tensor-bound: 4 B H Tc L D flops per call."""
    import torch
    from gated_deltanet_linear_chunked_b200 import workloads as wl
    w = wl.sink_window_stream()
    gen = torch.Generator(device=dev).manual_seed(17)
    shape = (w.B, w.Tc, w.H, w.D)
    cshape = (w.B, w.n_sink + w.window, w.Tc, w.H, w.D)
    sets = []
    for _ in range(3):
        x = {n: torch.randn(shape, generator=gen, device=dev).to(torch.bfloat16) for n in "qkv"}
        x["kc"] = torch.randn(cshape, generator=gen, device=dev).to(torch.bfloat16)
        x["vc"] = torch.randn(cshape, generator=gen, device=dev).to(torch.bfloat16)
        x["out"] = torch.empty(shape, dtype=torch.bfloat16, device=dev)
        sets.append(x)
    c = 5
    nkeys = len([m for m in range(c + 1) if m < w.n_sink or m > c - w.window]) * w.Tc

    def call(i):
        x = sets[i % len(sets)]
        gdn.sink_window_attention(x["q"], x["k"], x["v"], x["kc"], x["vc"], c, w.n_sink, w.window,
                                  out=x["out"], stream=stream)
    with torch.cuda.stream(stream):
        for i in range(6):
            call(i)
    barrier()
    reps = 30
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        for i in range(reps):
            call(i)
    e1.record(stream)
    barrier()
    ms = e0.elapsed_time(e1) / reps

    def direct(i):
        with torch.cuda.stream(stream):
            call(i)
    split = kernel_times(lib, direct, 6, 1)
    flops = 4 * w.B * w.H * w.Tc * nkeys * w.D
    chunk_bytes = w.B * w.Tc * w.H * w.D * 2
    nbytes = chunk_bytes * (4 + 2 * (nkeys // w.Tc - 1) + 2)   # q k v out, cache reads, cache writes
    tf = flops / (ms / 1000.0) / 1e12
    kms = split.get("gdn_sink_window_kernel", {}).get("ms_per_launch", ms)
    return {"workload": f"{w.name} (B{w.B} H{w.H} D{w.D} Tc{w.Tc}, n_sink {w.n_sink}, "
                        f"window {w.window}, chunk {c}: {nkeys} keys)",
            "ms_per_call": ms, "head_tokens_per_s": w.B * w.H * w.Tc / (ms / 1000.0),
            "kernels": split,
            "roofline": {"bound": "tensor", "achieved": tf, "unit": "TFLOP/s",
                         "peak": peaks["bf16_tflops"], "frac": tf / peaks["bf16_tflops"],
                         "kernel_tflops": flops / (kms / 1000.0) / 1e12,
                         "kernel_frac": flops / (kms / 1000.0) / 1e12 / peaks["bf16_tflops"],
                         "algorithmic_flops": flops, "algorithmic_bytes": nbytes,
                         "hbm_floor_us": 1e6 * nbytes / (peaks["hbm_gbs"] * 1e9),
                         "tensor_floor_us": 1e6 * flops / (peaks["bf16_tflops"] * 1e12),
                         "peak_source": f"{peak_kind} bf16_tflops (burst: the kernel is timed alone)"}}


def roofline_times(w, bidir, peaks):
    """Seconds the step would take at the HBM and at the tensor-pipe peak:
    algorithmic bytes over the measured copy bandwidth, chunked-form FLOPs
    over the sustained bf16 GEMM rate (the roofline definition the scope
    table fixes)."""
    return (algorithmic_bytes(w) / (peaks["hbm_gbs"] * 1e9),
            algorithmic_flops(w, bidir) / (peaks["bf16_tflops_sustained"] * 1e12))


def roofline_of(w, kernels, ms_per_step, peaks, peak_kind, bidir):
    """The dominant kernel against the path's binding bound: achieved = the
    path's algorithmic bytes (or FLOPs) per step -- one launch of each kernel
    processes every unit of the step -- over that kernel's mean launch time.
    `path` gives the same figure over the whole step's time."""
    bytes_step = algorithmic_bytes(w)
    flops_step = algorithmic_flops(w, bidir)
    dom = max(kernels, key=lambda k: kernels[k]["ms_per_launch"])
    dom_ms = kernels[dom]["ms_per_launch"]
    t_hbm, t_tc = roofline_times(w, bidir, peaks)
    if t_tc > t_hbm:
        bound, unit, work = "tensor", "TFLOP/s", flops_step / 1e12
        peak = peaks["bf16_tflops_sustained"]
        src = f"{peak_kind} bf16_tflops_sustained"
    else:
        bound, unit, work, peak = "hbm", "GB/s", bytes_step / 1e9, peaks["hbm_gbs"]
        src = f"{peak_kind} hbm_gbs"
    achieved = work / (dom_ms / 1000.0)
    path_achieved = work / (ms_per_step / 1000.0)
    return {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
            "frac": achieved / peak, "traffic": recorded_traffic(dom),
            "traffic_source": "committed ncu summary profiles/dram_traffic.txt, valid while the "
                              "kernel's source hash matches (else null)",
            "peak_source": src, "kernel": dom,
            "algorithmic_bytes_per_launch": bytes_step, "algorithmic_flops_per_launch": flops_step,
            "ms_per_launch": dom_ms, "kernels": kernels,
            "kernel_share_frac": {k: (kernel_algorithmic_bytes(k, w) / (v["ms_per_launch"] / 1000.0)
                                      / 1e9 / peaks["hbm_gbs"]) for k, v in kernels.items()},
            "path": {"ms_per_step": ms_per_step, "achieved": path_achieved, "frac": path_achieved / peak,
                     "roofline_us": 1e6 * max(t_hbm, t_tc),
                     "algorithmic_bytes": bytes_step, "algorithmic_flops": flops_step,
                     "achieved_gbs": bytes_step / (ms_per_step / 1000.0) / 1e9,
                     "achieved_tflops": flops_step / (ms_per_step / 1000.0) / 1e12,
                     "hbm_frac": bytes_step / (ms_per_step / 1000.0) / 1e9 / peaks["hbm_gbs"],
                     "tensor_frac_of_sustained": flops_step / (ms_per_step / 1000.0) / 1e12
                     / peaks["bf16_tflops_sustained"]}}


def main():
    args = parse()
    from gated_deltanet_linear_chunked_b200 import workloads as wl
    w = wl.stream_chunk(args.mode)
    if args.impl == "reference":
        return run_reference(args, w)

    import torch
    import torch.distributed as dist
    import gated_deltanet_linear_chunked_b200 as gdn
    from gated_deltanet_linear_chunked_b200 import _lib

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    lib = _lib.load()
    stream = torch.cuda.Stream(device=dev)
    fn = gdn.chunk_bidir if w.mode == "bidir" else gdn.chunk_fwd
    use_graph = not args.no_graph

    # ---- inputs: one seeded chunk per rank, copied into N_SETS rotating sets
    w_r = rank_workload(w, rank)
    xh = wl.make_inputs(w_r)
    base, sets = make_sets(w, xh, dev, N_SETS)
    torch.cuda.synchronize()

    # launches per step (counted on a direct call)
    c0 = lib.gdn_launch_count()
    with torch.cuda.stream(stream):
        fn(sets[0]["q"], sets[0]["k"], sets[0]["v"], sets[0]["g"], sets[0]["beta"],
           sets[0]["state_in"], state_out=sets[0]["state_out"], out=sets[0]["out"],
           chunk=w.chunk, stream=stream)
    launches_per_step = lib.gdn_launch_count() - c0
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])
        torch.cuda.synchronize()

    main_run = Stepper(fn, sets, stream, w.chunk, use_graph)
    with nvtx("warmup"):
        main_run.warm(max(3, args.warmup))
    barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    try:
        nvml_index = torch.cuda._get_nvml_device_index(local)
    except Exception:
        nvml_index = local
    with ClockSampler(nvml_index) as clocks, nvtx("timed"):
        barrier()
        ev0.record(stream)
        main_run.run(args.steps)
        ev1.record(stream)
        barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    ms_per_step = ms / args.steps
    value = job_throughput(world, args.steps, w.head_tokens, ms)
    main_run.release()

    # ---- end to end through the public API: pinned host -> device, call, device -> host.
    # Every step copies its inputs in and its results out.  Three streams
    # (copy-in, the compute stream, copy-out) over the N_SETS device sets let
    # step i + 1's inputs load while step i computes and step i - 1's results
    # return, as a streaming server would; a set is reused only after its
    # previous results have left.
    e2e_steps = max(3, min(args.steps, 200))
    host = {n: (t.cpu().pin_memory()) for n, t in base.items()}
    host_res = [(torch.empty((w.B, w.T, w.H, w.Dv), dtype=torch.bfloat16).pin_memory(),
                 torch.empty_like(host["state_in"]).pin_memory()) for _ in range(N_SETS)]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in host_res[0])
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(N_SETS)]
    ev_done = [torch.cuda.Event() for _ in range(N_SETS)]
    ev_out = [torch.cuda.Event() for _ in range(N_SETS)]
    used = [False] * N_SETS

    def e2e_step(i):
        k = i % N_SETS
        s = sets[k]
        if used[k]:
            s_in.wait_event(ev_out[k])  # the set's previous results have left
        with torch.cuda.stream(s_in):
            for n in ("q", "k", "v", "g", "beta", "state_in"):
                s[n].copy_(host[n], non_blocking=True)
            ev_in[k].record(s_in)
        stream.wait_event(ev_in[k])
        fn(s["q"], s["k"], s["v"], s["g"], s["beta"], s["state_in"], state_out=s["state_out"],
           out=s["out"], chunk=w.chunk, stream=stream)
        ev_done[k].record(stream)
        s_out.wait_event(ev_done[k])
        with torch.cuda.stream(s_out):
            host_res[k][0].copy_(s["out"], non_blocking=True)
            host_res[k][1].copy_(s["state_out"], non_blocking=True)
            ev_out[k].record(s_out)
        used[k] = True

    with nvtx("e2e"):
        for i in range(max(3, N_SETS)):
            e2e_step(i)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        for i in range(e2e_steps):
            e2e_step(i)
        e1.record(s_out)
        barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = job_throughput(world, e2e_steps, w.head_tokens, e2e_ms)

    # ---- per-kernel device times and the roofline of the dominant kernel
    peaks, peak_kind = load_peaks()
    n_prof = max(3, min(args.steps, 100))

    def direct(i):
        with torch.cuda.stream(stream):
            main_run.call(i)
    kernels = kernel_times(lib, direct, n_prof, launches_per_step)
    roofline = roofline_of(w, kernels, ms_per_step, peaks, peak_kind, w.mode == "bidir")

    # ---- side figures: the other mode (its own roofline), and the 15-layer
    # stacked stream (direct calls and one captured graph)
    extras = {}
    chosen = set() if args.no_extras else (
        {"side", "long", "backward", "sink_window"} if args.extras == "all"
        else {x.strip() for x in args.extras.split(",") if x.strip()})
    if "side" in chosen:
        other = "bidir" if w.mode == "fwd" else "fwd"
        fo = gdn.chunk_bidir if other == "bidir" else gdn.chunk_fwd
        n_side = max(3, min(args.steps, 200))
        with nvtx(f"{other}_chunk"):
            side = Stepper(fo, sets, stream, w.chunk, use_graph)
            side.warm(max(3, args.warmup))
            barrier()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            side.run(n_side)
            a1.record(stream)
            barrier()
            side.release()
        other_ms = a0.elapsed_time(a1) / n_side

        def side_direct(i):
            with torch.cuda.stream(stream):
                side.call(i)
        side_kernels = kernel_times(lib, side_direct, n_prof, launches_per_step)
        wo = wl.stream_chunk(other)
        extras[f"{other}_chunk"] = {
            "workload": wo.name, "ms_per_step": other_ms,
            "head_tokens_per_s": w.head_tokens / (other_ms / 1000.0),
            "latent_frames_per_s": w.B * (w.T / 880) / (other_ms / 1000.0),
            "steps": n_side, "timing": "CUDA graph replays" if use_graph else "direct calls",
            "roofline": roofline_of(wo, side_kernels, other_ms, peaks, peak_kind, other == "bidir")}
        # 32 chunks x 15 layers in model order (chunk-major), one state per
        # layer carried in place, inputs rotating over the sets; the pages'
        # streaming GDN is bidirectional, the causal stack is reported too
        n_chunks = 32
        for smode, sfn in (("bidir", gdn.chunk_bidir), ("causal", gdn.chunk_fwd)):
            states = [torch.zeros_like(base["state_in"]) for _ in range(wl.GDN_LAYERS)]

            def stack_calls():
                i = 0
                for _c in range(n_chunks):
                    for l in range(wl.GDN_LAYERS):
                        s = sets[i % N_SETS]
                        sfn(s["q"], s["k"], s["v"], s["g"], s["beta"], states[l],
                            state_out=states[l], out=s["out"], chunk=w.chunk, stream=stream)
                        i += 1
            res = {"calls": n_chunks * wl.GDN_LAYERS}
            frames = n_chunks * 3
            with nvtx(f"stack_{smode}"), torch.cuda.stream(stream):
                stack_calls()
                barrier()
                b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                b0.record(stream)
                stack_calls()
                b1.record(stream)
                barrier()
                res["direct_ms"] = b0.elapsed_time(b1)
                res["direct_latent_frames_per_s"] = frames / (res["direct_ms"] / 1000.0)
                if use_graph:
                    gs = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(gs, stream=stream):
                        stack_calls()
                    for _ in range(2):
                        gs.replay()
                    barrier()
                    b0.record(stream)
                    reps = 3
                    for _ in range(reps):
                        gs.replay()
                    b1.record(stream)
                    barrier()
                    res["graph_ms"] = b0.elapsed_time(b1) / reps
                    res["graph_latent_frames_per_s"] = frames / (res["graph_ms"] / 1000.0)
                    del gs
            ws = wl.stream_chunk("bidir" if smode == "bidir" else "fwd")
            res["bound_latent_frames_per_s"] = frames / (res["calls"] * max(
                roofline_times(ws, smode == "bidir", peaks)))
            extras[f"stack_32x15_{smode}"] = res
        # the fused gate prologue: the causal chunk with the gate layer's bf16
        # logits as inputs (own input sets, graph-timed like the main figure)
        wlg = wl.stream_chunk_logits("fwd", seed=w_r.seed)
        _, lsets = make_sets(wlg, wl.make_inputs(wlg), dev, N_SETS)
        with nvtx("fwd_logits_chunk"):
            lg = Stepper(gdn.chunk_fwd_logits, lsets, stream, w.chunk, use_graph, gate_keys(wlg))
            lg.warm(max(3, args.warmup))
            barrier()
            a0.record(stream)
            lg.run(n_side)
            a1.record(stream)
            barrier()
            lg.release()
        lg_ms = a0.elapsed_time(a1) / n_side

        def lg_direct(i):
            with torch.cuda.stream(stream):
                lg.call(i)
        extras["fwd_logits_chunk"] = {
            "workload": wlg.name, "ms_per_step": lg_ms,
            "head_tokens_per_s": w.head_tokens / (lg_ms / 1000.0), "steps": n_side,
            "timing": "CUDA graph replays" if use_graph else "direct calls",
            "roofline": roofline_of(wlg, kernel_times(lib, lg_direct, n_prof, launches_per_step),
                                    lg_ms, peaks, peak_kind, False)}
        del lsets
    if "long" in chosen:
        extras.update(long_stream_figures(gdn, lib, w, stream, dev, peaks, peak_kind, barrier))
    if "backward" in chosen:
        extras["bidir_backward_chunk"] = backward_figure(gdn, lib, base, w, stream, peaks, peak_kind,
                                                         barrier)
    if "sink_window" in chosen:
        extras["sink_window_chunk"] = sink_window_figure(gdn, lib, stream, dev, peaks, peak_kind,
                                                         barrier)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        with nvtx("cpu_baseline"):
            cpu = cpu_baseline(w, args.cpu_seconds)

    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "Dk": w.Dk, "Dv": w.Dv,
                   "chunk": w.chunk, "mode": w.mode, "io": "bf16 q/k/v/out, fp32 g/beta/state",
                   "l2": f"inputs rotate over {N_SETS} sets of "
                         f"{algorithmic_bytes(w) / 1e6:.1f} MB "
                         f"({N_SETS * algorithmic_bytes(w) / 1e6:.0f} MB > 126 MB L2)",
                   "graph": use_graph,
                   "warmup_replays": max(3, args.warmup, N_SETS) if use_graph else max(3, args.warmup),
                   "parallelism": f"replicas x{world} (independent chunk streams)"},
        "latent_frames_per_s": value / (w.B * w.H * 880),
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "pipelining": "copy-in / compute / copy-out on three streams over the "
                              f"{N_SETS} device sets"},
        "gpu_launches": int(launches_per_step * args.steps),
        "launches_per_step": int(launches_per_step),
        "clocks": clocks.summary(),
        "extras": extras,
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
