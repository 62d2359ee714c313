"""Benchmark of the key-gated GLA forward on B200: tokens/s and % of roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload batched] [--schedule auto|fused|three_phase]

A step is one full GLA forward (every phase of the chunkwise operator) over
one batch of the workload; steps alternate the workload's scan directions.
Inputs are seeded synthetic tensors resident in HBM before the timed region;
they are larger than L2, so no flush is needed between steps.  Timing uses
CUDA events on the launching stream, W untimed warm-up steps, then exactly K
timed steps bracketed by a barrier and a device synchronize; with N ranks
(torchrun, one process per GPU) every rank runs its own batch (weak scaling,
no collective on the data path) and the max time over ranks is reported.
Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle (the only reference that exists:
the pages publish no code) on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
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

from recurrent_vision_backbone_key_b200 import gtr_gla  # noqa: E402
from recurrent_vision_backbone_key_b200.synthetic import (  # noqa: E402
    SSWIGLU_WORKLOADS, WORKLOADS, make_sswiglu_inputs, make_workload_inputs)
from recurrent_vision_backbone_key_b200 import dist as rdist  # noqa: E402

METRIC = "GLA forward tokens/s and % of roofline (HBM GB/s or TC util) at 1 B200"
DIR_NAMES = ["L2R", "R2L", "T2B", "B2T"]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


# Committed ncu summaries: (file, kernel sources hashed into it) per kernel.
PROFILE_SUMMARIES = {
    "gla_walk_kernel<64,WALK_SEQ>": ("gla_walk_d64_batched.md",
                                     ("gla_walk.cuh", "gla_tcgen05.cuh", "gla_tc.cuh", "gla_common.cuh")),
    "gla_umma_kernel": ("gla_umma_fused_d64_batched.md",
                        ("gla_umma.cuh", "gla_tcgen05.cuh", "gla_tc.cuh", "gla_common.cuh")),
    "gla_tc_kernel<64,64,FUSED,1>": ("gla_tc_fused_d64_batched.md", ("gla_tc.cuh", "gla_common.cuh")),
}


def planned_kernel(w, schedule):
    """(plan code, kernel name) of what the library launches for this workload
    and schedule on this device (the library's own dispatch, gtr_gla_plan)."""
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    plan = gtr_gla.gtr_gla_plan(w.B, w.heads, w.grid_h, w.grid_w, w.d_k, w.d_v, w.chunk, schedule, sms)
    names = {0: "three-phase (summary, scan, output)", 1: "three-phase on CUDA cores",
             2: f"gla_tc_kernel<{w.d_k},{w.d_v},FUSED,1>", 3: f"gla_tc_kernel<{w.d_k},{w.d_v},FUSED,2>",
             4: "gla_umma_kernel", 5: f"gla_walk_kernel<{w.d_k},WALK_SEQ>",
             6: "three-phase, mma.sync phases (summary, scan, output)"}
    return plan, names.get(plan, "unknown")


def profiled_traffic(w, kernel):
    """DRAM bytes per launch of the given kernel from the committed ncu summary,
    if that summary was taken on this workload from the current kernel source."""
    import hashlib
    if w.name != "batched" or kernel not in PROFILE_SUMMARIES:
        return None
    fname, sources = PROFILE_SUMMARIES[kernel]
    prof = os.path.join(ROOT, "profiles", fname)
    if not os.path.exists(prof):
        return None
    src = os.path.join(ROOT, "recurrent_vision_backbone_key_b200", "csrc")
    h = hashlib.sha256()
    for f in sources:
        with open(os.path.join(src, f), "rb") as fh:
            h.update(fh.read())
    fields = {}
    for line in open(prof):
        if ":" in line and line.split(":")[0].strip() in ("kernel_source_sha256_16", "traffic_bytes_per_launch"):
            k, v = line.split(":", 1)
            fields[k.strip()] = v.strip()
    if fields.get("kernel_source_sha256_16") != h.hexdigest()[:16]:
        return None
    return int(fields["traffic_bytes_per_launch"])


def graph_replay_ms(call, dirs, replays=50):
    """Median CUDA-event milliseconds of one forward replayed from a CUDA graph
    (one graph per direction, replayed in turn)."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for d in dirs:  # the workspaces of this stream exist before the capture
            call(d, side)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graphs = []
    for d in dirs:
        gph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gph, stream=side):
            call(d, side)
        graphs.append(gph)
    for i in range(3 * len(graphs)):
        graphs[i % len(graphs)].replay()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(replays)]
    torch.cuda.synchronize()
    for i, (a, b) in enumerate(ev):
        a.record()
        graphs[i % len(graphs)].replay()
        b.record()
    torch.cuda.synchronize()
    t = sorted(a.elapsed_time(b) for a, b in ev)
    del graphs
    return {"median_ms_per_forward": t[len(t) // 2], "min_ms": t[0], "replays": replays,
            "note": "CUDA-graph replay, one forward per graph, CUDA events around each replay"}


def describe(w):
    dirs = "+".join(DIR_NAMES[d] for d in w.directions)
    return (f"{w.name}: B{w.B} {w.grid_h}x{w.grid_w} grid ({w.N} tokens), {w.heads} heads, "
            f"d_k={w.d_k} d_v={w.d_v}, chunk {w.chunk}, {w.gate} gates, directions {dirs} "
            f"alternating per step")


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index, period_s=0.005):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self.ok = False
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.nvml = None

    def _sample(self):
        try:
            self.samples.append(self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM))
            self.reasons |= int(self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.h))
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._sample()
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()
            self._sample()

    def summary(self):
        if not self.ok or not self.samples:
            return None
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": float(self.max_mhz),
                "samples": len(self.samples), "reasons": names}


def oracle_rate(w, q, k, v, g, budget_s, nthreads, directions):
    """Times the fp64 oracle on (b, h) sequences of the workload until about
    budget_s seconds of CPU work; returns (tokens/s, sample description)."""
    from oracle import oracle
    oracle.build()
    rng = np.random.default_rng(0)
    picks = [(int(b), int(h)) for b, h in zip(rng.integers(w.B, size=4096), rng.integers(w.heads, size=4096))]
    done_th, elapsed, n_seq, i = 0, 0.0, 0, 0
    batch = max(1, nthreads)
    while elapsed < budget_s and n_seq < len(picks):
        sel = picks[n_seq:n_seq + batch]
        # gather the selected sequences as one [n, N, 1, d] problem
        take = lambda x: torch.stack([x[b, :, h:h + 1, :] for b, h in sel]).cpu()
        qs, ks, vs, gs = take(q), take(k), take(v), take(g)
        d = directions[i % len(directions)]
        t0 = time.perf_counter()
        oracle.gla_serial(qs, ks, vs, gs, w.grid_h, w.grid_w, d, nthreads=nthreads)
        elapsed += time.perf_counter() - t0
        done_th += len(sel) * w.N
        n_seq += len(sel)
        i += 1
        batch = max(batch, int(batch * min(4.0, 0.5 * budget_s / max(elapsed, 1e-3))))
        batch = min(batch, 64 * max(1, nthreads))
    tokens_per_s = done_th / elapsed  # one head of one token per unit; heads run in parallel
    tokens_per_s /= w.heads  # a token is complete once all its heads are
    sample = (f"{n_seq} (batch, head) sequences of {w.N} tokens drawn from the workload, "
              f"serial fp64 recurrence, {elapsed:.1f} s")
    return tokens_per_s, sample


def run_reference(args, w):
    rank, world = rdist.rank_world()
    if rank != 0:
        return 0
    q, k, v, g = make_workload_inputs(w, seed=0, device="cpu")
    nthreads = os.cpu_count() or 1
    from oracle import oracle
    oracle.build()
    rng = np.random.default_rng(1)
    per_step = max(1, nthreads)
    def step(i):
        sel = [(int(rng.integers(w.B)), int(rng.integers(w.heads))) for _ in range(per_step)]
        take = lambda x: torch.stack([x[b, :, h:h + 1, :] for b, h in sel])
        oracle.gla_serial(take(q), take(k), take(v), take(g), w.grid_h, w.grid_w,
                          w.directions[i % len(w.directions)], nthreads=nthreads)
        return len(sel) * w.N
    for i in range(args.warmup):
        step(i)
    th = 0
    t0 = time.perf_counter()
    for i in range(args.steps):
        th += step(i)
    dt = time.perf_counter() - t0
    value = th / w.heads / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": describe(w), "B": w.B, "grid": [w.grid_h, w.grid_w],
                   "heads": w.heads, "d_k": w.d_k, "d_v": w.d_v, "chunk": w.chunk,
                   "step": f"fp64 CPU oracle on {per_step} sampled (batch, head) sequences"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
                         "sample": f"{per_step} (batch, head) sequences of {w.N} tokens per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def time_steps(fn, steps, stream, flush=None):
    """Runs fn(i) for i in range(steps) on `stream`; ms.  Without `flush`, one
    pair of events brackets all steps.  With it, flush() runs before every
    step (outside the timing) and the per-step event times are summed."""
    if flush is None:
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for i in range(steps):
            fn(i)
        end.record(stream)
        end.synchronize()
        return start.elapsed_time(end)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i, (a, b) in enumerate(ev):
        flush()
        a.record(stream)
        fn(i)
        b.record(stream)
    ev[-1][1].synchronize()
    return sum(a.elapsed_time(b) for a, b in ev)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="batched", choices=sorted(WORKLOADS) + sorted(SSWIGLU_WORKLOADS))
    ap.add_argument("--schedule", default="auto", choices=sorted(gtr_gla.SCHEDULES))
    ap.add_argument("--dtype", default="f16", choices=["f16", "bf16"],
                    help="element type of q, k, v and out (bf16: gtr_gla_forward_bf16)")
    ap.add_argument("--variant", default="plain", choices=["plain", "gated", "state"],
                    help="gated: output gate on the RMS-normalised output (gtr_gla_forward_gated); "
                         "state: initial state in, final state out (gtr_gla_forward_state)")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-graph", action="store_true", help="skip the CUDA-graph replay timing")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.workload in SSWIGLU_WORKLOADS:
        return run_sswiglu(args, SSWIGLU_WORKLOADS[args.workload])
    w = WORKLOADS[args.workload]

    if args.impl == "reference":
        return run_reference(args, w)

    rank, world = rdist.init_from_env(backend="nccl")
    dev = rdist.local_device()
    torch.cuda.set_device(dev)
    lib = gtr_gla.load()
    stream = torch.cuda.current_stream()
    sched = gtr_gla.SCHEDULES[args.schedule]

    tdtype = torch.bfloat16 if args.dtype == "bf16" else torch.float16
    if args.dtype == "bf16" and args.variant != "plain":
        raise SystemExit("--dtype bf16 runs the plain forward only")
    q, k, v, g = make_workload_inputs(w, seed=rank, device=f"cuda:{dev}", dtype=tdtype)
    out = torch.empty((w.B, w.N, w.heads, w.d_v), dtype=tdtype, device=f"cuda:{dev}")
    dirs = list(w.directions)
    extra_bytes = 0  # algorithmic bytes of the variant beyond the forward's
    if args.variant == "gated":
        gate = torch.randn((w.B, w.N, w.heads, w.d_v), device=f"cuda:{dev}").to(torch.float16)
        norm_w = torch.ones(w.d_v, device=f"cuda:{dev}")
        extra_bytes = w.token_heads * 2 * w.d_v  # the gate read
    if args.variant == "state":
        S0 = torch.randn((w.B, w.heads, w.d_k, w.d_v), device=f"cuda:{dev}") * 0.1
        SN = torch.empty_like(S0)
        extra_bytes = 2 * S0.numel() * 4  # S_0 read, S_N written

    def step(i):
        d = dirs[i % len(dirs)]
        if args.dtype == "bf16":
            st = gtr_gla.gtr_gla_forward_bf16(q, k, v, g, w.B, w.heads, w.grid_h, w.grid_w, w.d_k, w.d_v, d,
                                              w.chunk, out, stream)
        elif args.variant == "gated":
            st = gtr_gla.gtr_gla_forward_gated(q, k, v, g, gate, norm_w, 1e-5, w.B, w.heads, w.grid_h, w.grid_w,
                                               w.d_k, w.d_v, d, w.chunk, out, stream)
        elif args.variant == "state":
            st = gtr_gla.gtr_gla_forward_state(q, k, v, g, S0, w.B, w.heads, w.grid_h, w.grid_w, w.d_k, w.d_v, d,
                                               w.chunk, out, SN, stream)
        else:
            st = gtr_gla.gtr_gla_forward_ex(q, k, v, g, w.B, w.heads, w.grid_h, w.grid_w, w.d_k, w.d_v, d,
                                            w.chunk, sched, out, stream)
        gtr_gla.check(st)

    # Inputs smaller than twice L2 would be read from L2 by the next step:
    # then L2 is flushed (a write larger than L2) before every timed step.
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = None
    if alg_bytes_total(w) < 2 * l2:
        scrub = torch.empty(2 * l2, dtype=torch.uint8, device=f"cuda:{dev}")
        flush = lambda: scrub.fill_(1)
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    rdist.barrier()
    l0 = gtr_gla.gtr_gla_launch_count()
    with ClockSampler(dev) as clocks:
        torch.cuda.synchronize()
        ms = time_steps(step, args.steps, stream, flush)
        torch.cuda.synchronize()
    launches = gtr_gla.gtr_gla_launch_count() - l0
    rdist.barrier()
    assert gtr_gla.gtr_gla_get_last_device_status(stream) == 0
    ms_max = rdist.max_over_ranks(ms)
    tokens_all = float(w.B * w.N * args.steps * world)
    value = tokens_all / (ms_max * 1e-3)

    # Roofline: the forward's algorithmic bytes (q, k, v, out in fp16, g in
    # fp32, each once) over the time of one whole forward.  With one kernel
    # per step that is also the dominant kernel's launch time; the
    # three-phase schedule's per-phase times are reported beside it, their
    # chunk-state traffic counts as overhead, not as work.
    hbm_peak, tc_peak, peak_kind = measured_peaks()
    alg_bytes = w.algorithmic_bytes() + extra_bytes
    per_forward_ms = ms / args.steps
    plan, dominant = planned_kernel(w, args.schedule)
    if args.dtype == "bf16" or args.variant != "plain":  # these entry points always run the walk kernel
        plan = 5
        dominant = (f"gla_walk_kernel<{w.d_k},WALK_SEQ>" + (",gated" if args.variant == "gated" else "")
                    + (",bf16" if args.dtype == "bf16" else ""))
    phase_ms = None
    if plan in (0, 1, 6):  # three phases: time them one by one as well
        phase_ms = time_phases(w, q, k, v, g, out, stream, max(3, min(args.steps, 50)))
    achieved = alg_bytes / (per_forward_ms * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak,
                "traffic": profiled_traffic(w, dominant) if phase_ms is None else None,
                "kernel": dominant, "peak_kind": f"{peak_kind} hbm_gbs (copy, burst)",
                "algorithmic_bytes_per_launch": alg_bytes,
                "tensor_flops_per_step": w.algorithmic_flops(),
                "tensor_frac_of_bf16_peak": w.algorithmic_flops() / (per_forward_ms * 1e-3) / 1e12 / tc_peak}
    if phase_ms:
        roofline["phase_ms"] = phase_ms
        roofline["note"] = ("frac is the whole forward (three launches); phase_ms are the phases "
                            "timed one by one")

    # The pages' latency protocol: median CUDA-event time of one forward
    # replayed from a CUDA graph (outside the timed region above).
    graph = None
    if not args.no_graph and args.dtype == "f16" and args.variant == "plain":
        graph = graph_replay_ms(lambda d, st: gtr_gla.check(gtr_gla.gtr_gla_forward_ex(
            q, k, v, g, w.B, w.heads, w.grid_h, w.grid_w, w.d_k, w.d_v, d, w.chunk, sched, out, st)), dirs)

    # End to end through the host-buffer entry point: pinned host inputs in,
    # host output back, every step.
    e2e = None
    if args.e2e_steps > 0 and args.dtype == "f16" and args.variant == "plain":
        qh, kh, vh, gh = (x.cpu().pin_memory() for x in (q, k, v, g))
        oh = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        def e2e_step(i):
            gtr_gla.check(gtr_gla.gtr_gla_forward_host(qh, kh, vh, gh, w.B, w.heads, w.grid_h,
                                                       w.grid_w, w.d_k, w.d_v, dirs[i % len(dirs)],
                                                       w.chunk, oh, stream))
        e2e_step(0)
        torch.cuda.synchronize()
        rdist.barrier()
        t0 = time.perf_counter()
        for i in range(args.e2e_steps):
            e2e_step(i)
        torch.cuda.synchronize()
        e2e_s = rdist.max_over_ranks(time.perf_counter() - t0)
        h2d = sum(x.numel() * x.element_size() for x in (q, k, v, g))
        d2h = out.numel() * out.element_size()
        e2e = {"value": float(w.B * w.N * args.e2e_steps * world / e2e_s), "unit": "tokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": args.e2e_steps, "timer": "host wall clock around synchronous calls"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        nthreads = os.cpu_count() or 1
        val, sample = oracle_rate(w, q, k, v, g, args.cpu_budget, nthreads, dirs)
        cpu = {"value": val, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
               "sample": sample}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": args.dtype,
            "data": "synthetic",
            "config": {"workload": describe(w), "B": w.B, "grid": [w.grid_h, w.grid_w],
                       "heads": w.heads, "d_k": w.d_k, "d_v": w.d_v, "chunk": w.chunk,
                       "schedule": args.schedule, "variant": args.variant,
                       "parallelism": f"dp{world} (independent batches)",
                       "l2": (f"inputs larger than L2 ({alg_bytes_total(w) / 1e6:.0f} MB per step), no flush"
                              if flush is None else
                              f"L2 flushed before every timed step ({2 * l2 / 1e6:.0f} MB write, outside the "
                              f"per-step CUDA events); {alg_bytes_total(w) / 1e6:.1f} MB per step")},
            "token_heads_per_s": value * w.heads,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "graph": graph,
            "gpu_launches": int(launches), "clocks": clocks.summary(),
        }
        print(json.dumps(line), flush=True)
    rdist.finalize()
    return 0


def run_sswiglu(args, wl):
    """Spatial SwiGLU gating with the fused 3x3 depthwise convolution: one
    gtr_sswiglu_forward call per step over the workload's [B, H*W, C] branches."""
    rank, world = rdist.init_from_env(backend="nccl")
    dev = rdist.local_device()
    torch.cuda.set_device(dev)
    gtr_gla.load()
    stream = torch.cuda.current_stream()
    a, v, wc, bias = make_sswiglu_inputs(wl.B, wl.grid_h, wl.grid_w, wl.C, seed=rank, device=f"cuda:{dev}")
    out = torch.empty_like(a)

    def step(i):
        gtr_gla.check(gtr_gla.gtr_sswiglu_forward(a, v, wc, bias, wl.B, wl.grid_h, wl.grid_w, wl.C, out, stream))

    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = None
    if wl.algorithmic_bytes() < 2 * l2:
        scrub = torch.empty(2 * l2, dtype=torch.uint8, device=f"cuda:{dev}")
        flush = lambda: scrub.fill_(1)
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    rdist.barrier()
    l0 = gtr_gla.gtr_gla_launch_count()
    with ClockSampler(dev) as clocks:
        torch.cuda.synchronize()
        ms = time_steps(step, args.steps, stream, flush)
        torch.cuda.synchronize()
    launches = gtr_gla.gtr_gla_launch_count() - l0
    rdist.barrier()
    ms_max = rdist.max_over_ranks(ms)
    value = float(wl.B * wl.N * args.steps * world) / (ms_max * 1e-3)
    hbm_peak, _, peak_kind = measured_peaks()
    achieved = wl.algorithmic_bytes() / (ms / args.steps * 1e-3) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak,
                "traffic": None, "kernel": "sswiglu_kernel", "peak_kind": f"{peak_kind} hbm_gbs (copy, burst)",
                "algorithmic_bytes_per_launch": wl.algorithmic_bytes()}
    e2e = None
    if args.e2e_steps > 0:
        ah, vh = a.cpu().pin_memory(), v.cpu().pin_memory()
        oh = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        def e2e_step():
            a.copy_(ah, non_blocking=True)
            v.copy_(vh, non_blocking=True)
            step(0)
            oh.copy_(out, non_blocking=True)
            torch.cuda.current_stream().synchronize()
        e2e_step()
        rdist.barrier()
        t0 = time.perf_counter()
        for _ in range(args.e2e_steps):
            e2e_step()
        e2e_s = rdist.max_over_ranks(time.perf_counter() - t0)
        e2e = {"value": float(wl.B * wl.N * args.e2e_steps * world / e2e_s), "unit": "tokens/s",
               "h2d_bytes_per_step": int(2 * a.numel() * 2), "d2h_bytes_per_step": int(out.numel() * 2),
               "steps": args.e2e_steps, "timer": "host wall clock around copies in, the call, the copy out"}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle import oracle
        oracle.build()
        ac, vc, wcc, bc = a.cpu(), v.cpu(), wc.cpu(), bias.cpu()
        t0, n = time.perf_counter(), 0
        while time.perf_counter() - t0 < min(args.cpu_budget, 10.0) and n < wl.B:
            oracle.sswiglu(ac[n:n + 1], vc[n:n + 1], wcc, bc, wl.grid_h, wl.grid_w)
            n += 1
        dt = time.perf_counter() - t0
        cpu = {"value": n * wl.N / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
               "sample": f"{n} batch items of {wl.N} tokens x {wl.C} channels, fp64, one thread, {dt:.1f} s"}
    if rank == 0:
        line = {
            "metric": "S-SwiGLU gating (3x3 depthwise conv fused) tokens/s and % of HBM roofline at 1 B200",
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f16", "data": "synthetic",
            "config": {"workload": f"{wl.name}: B{wl.B} {wl.grid_h}x{wl.grid_w} grid, C={wl.C}",
                       "parallelism": f"dp{world} (independent batches)",
                       "l2": ("inputs larger than L2, no flush" if flush is None else "L2 flushed before every step")},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": int(launches),
            "clocks": clocks.summary(),
        }
        print(json.dumps(line), flush=True)
    rdist.finalize()
    return 0


def alg_bytes_total(w):
    return w.algorithmic_bytes()


def time_phases(w, q, k, v, g, out, stream, reps):
    nseq = w.B * w.heads
    nc = (w.N + w.chunk - 1) // w.chunk
    dS = torch.empty((nseq, nc, w.d_k, w.d_v), dtype=torch.float32, device=q.device)
    gam = torch.empty((nseq, nc, w.d_k), dtype=torch.float32, device=q.device)
    Se = torch.empty_like(dS)
    d = w.directions[0]
    calls = {
        "chunk_summary": lambda i: gtr_gla.check(gtr_gla.gtr_gla_chunk_summary(
            k, v, g, w.B, w.heads, w.grid_h, w.grid_w, w.d_k, w.d_v, d, w.chunk, dS, gam, stream)),
        "boundary_scan": lambda i: gtr_gla.check(gtr_gla.gtr_gla_boundary_scan(
            dS, gam, w.B, w.heads, nc, w.d_k, w.d_v, Se, stream)),
        "chunk_output": lambda i: gtr_gla.check(gtr_gla.gtr_gla_chunk_output(
            q, k, v, g, Se, w.B, w.heads, w.grid_h, w.grid_w, w.d_k, w.d_v, d, w.chunk, out,
            stream)),
    }
    res = {}
    for name, fn in calls.items():
        for i in range(3):
            fn(i)
        res[name] = time_steps(fn, reps, stream) / reps
    del dS, gam, Se
    return res


if __name__ == "__main__":
    sys.exit(main())
