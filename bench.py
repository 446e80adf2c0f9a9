#!/usr/bin/env python
"""Benchmark of the fused WTConv layer on B200: one step = forward +
input gradient + weight gradient over one synthetic batch.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload stage1|stage2|train_bf16|tiny]

With --gpus N > 1 and no torch.distributed environment, the script launches
itself as N ranks (torch.distributed.run, one rank per GPU, 127.0.0.1).

Prints one JSON line (rank 0).  Metric: modeled minimum HBM bytes of the three
calls divided by their device time (GB/s), the achieved fraction of the
measured HBM peak, and microseconds per call.  Modeled bytes per step:
6*N*e + 4*P (x read + y written, dy read + dx written, x and dy read; P the
float32 parameter bytes, read by every call and written once as gradients).

Timing: CUDA events on the launching stream around each call, after W warm-up
steps; L2 is flushed (a 256 MiB write) before every call; K steps between a
barrier + synchronize on both sides; the max over ranks.  With N > 1 every
rank runs its own batch (weak scaling) and the weight gradients are summed
over ranks with one NCCL all-reduce per step (data parallel).

`--impl reference` times the CPU oracle (the reference arm) on the host cores
on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "WTConv fwd+bwd HBM GB/s and % of 8 TB/s roofline; µs/call at WTConvNeXt shapes"
FALLBACK_HBM_GBS = 6650.0
SMS, FP32_LANES, MAX_SM_MHZ = 148, 128, 1965.0
L2_FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="stage1")
    ap.add_argument("--nhwc", action="store_true", help="channels-last (NHWC) activations for the named workload")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="time only the named workload (by default the other WTConvNeXt stage shapes are timed too)")
    ap.add_argument("--dist-check", action="store_true",
                    help="CPU check of the multi-rank launch path (gloo): each rank all-reduces synthetic weight "
                         "gradients and the slowest rank's time is reported; no kernels run")
    ap.add_argument("--compare", action="store_true",
                    help="time the unfused PyTorch layer and the plain depthwise conv beside this library "
                         "(context lines, not the bench line)")
    ap.add_argument("--compare-only", default="", help="with --compare: only the implementation named so")
    ap.add_argument("--profile-one-forward", action="store_true",
                    help="with --compare: run one forward per implementation between profiler start/stop")
    ap.add_argument("--sweep", action="store_true",
                    help="time the three calls at every point of the 128-point shape sweep (one JSON line each)")
    ap.add_argument("--sweep-steps", type=int, default=20, help="with --sweep: timed calls per point")
    ap.add_argument("--sweep-points", default="", help="with --sweep: one point index or a range, e.g. 5 or 0:32")
    return ap.parse_args()


# --------------------------------------------------------------------------
# Workload arithmetic (the modeled minimum traffic and the conv FMA count).
# --------------------------------------------------------------------------
def param_floats(c) -> int:
    return c.C * c.k * c.k * (1 + 4 * c.L) + 2 * c.C + 4 * c.L * c.C


def modeled_bytes(c) -> dict:
    N, e, P = c.numel, c.esize, 4 * param_floats(c)
    return {"fwd": 2 * N * e + P, "bwd_in": 2 * N * e + P, "bwd_w": 2 * N * e + 2 * P}


def conv_fmas(c) -> float:
    """Algorithmic multiply-adds of one call: base conv + every subband conv."""
    return c.numel * c.k * c.k * (1.0 + sum(4.0 ** -l for l in range(c.L)))


def workload_name(c, nhwc: bool = False) -> str:
    return (f"{c.name}: B={c.B} C={c.C} H={c.H} W={c.W} k={c.k} L={c.L} {c.dtype} {'NHWC' if nhwc else 'NCHW'}, "
            f"forward + backward_input + backward_weight")


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per launch of a
# kernel, from one ncu capture of the named workload (the command is in the
# named profile summary).  Each figure carries the SHA-256 of the kernel
# sources it was taken on; once those change it no longer describes the
# kernel and is reported as null.
KERNEL_SOURCES = ("wtconv_kernels.cuh", "wtconv_kinst.cuh", "wtconv_plan.h", "wtconv_planner.h",
                  "wtconv_launch.h", "wtconv_api.cu", "wtconv_k1.cu", "wtconv_k3.cu", "wtconv_k5.cu", "wtconv_k7.cu")
MEASURED_TRAFFIC = {
    # (workload, call): (bytes per launch, kernel, source digest, profile)
    ("stage1", "bwd_w"): (79442176.0, "wtconv_bwdw_partial_kernel",
                          "3955a401d12ac3da446d06c2d26f646631dd5e28b326d479e49c854035394e2e",
                          "profiles/wtconv_bwdw_partial_kernel_stage1.md"),
}


def kernel_source_digest() -> str:
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "memory_bound_cnn_wtconv_b200", "csrc", name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()


def measured_traffic(workload: str, call: str):
    ent = MEASURED_TRAFFIC.get((workload, call))
    if ent is None or ent[2] != kernel_source_digest():
        return None, None
    return ent[0], {"kernel": ent[1], "profile": ent[3]}


def hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# --------------------------------------------------------------------------
# Clock sampling during the timed region.
# --------------------------------------------------------------------------
class Clocks:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, enabled: bool, gpu_index: int):
        self.proc = None
        self.path = None
        self.gpu = gpu_index
        if enabled:
            try:
                fd, self.path = tempfile.mkstemp(suffix=".csv")
                os.close(fd)
                self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                              "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
                time.sleep(0.3)
            except Exception:
                self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8 or not f[0].isdigit() or int(f[0]) != self.gpu:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), f[4:8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for _, _, r in rows for i in range(4) if r[i].lower().startswith("active")})
        top = max(r[0] for r in rows)
        under_load = [r[0] for r in rows if r[0] >= 0.5 * top] or [r[0] for r in rows]
        return {"sm_mhz": statistics.median(under_load), "sm_max_mhz": rows[0][1], "reasons": reasons,
                "samples": len(rows)}


# --------------------------------------------------------------------------
# Distributed plumbing.
# --------------------------------------------------------------------------
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def allreduce_weight_grads(grads: dict, flat, dist) -> None:
    """Data parallel over the batch: sum the rank-local weight gradients over
    all ranks (one all-reduce of the flattened tensors) and write the sums
    back into `grads`."""
    import torch
    torch.cat([v.reshape(-1) for v in grads.values()], out=flat)
    dist.all_reduce(flat)
    off = 0
    for v in grads.values():
        n = v.numel()
        v.copy_(flat[off:off + n].view_as(v))
        off += n


def max_over_ranks(value: float, dist, device) -> float:
    """The slowest rank's value (timings are reported as the max over ranks)."""
    import torch
    t = torch.tensor([value], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def physical_gpu_index(local: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local < len(ids) and ids[local].isdigit():
            return int(ids[local])
    return local


# --------------------------------------------------------------------------
# CPU oracle timing (the reference arm and the reported CPU baseline).
# --------------------------------------------------------------------------
def oracle_sample(case, seconds: float, max_planes: int | None = None, wrap: bool = False):
    """Time the oracle's three calls on whole batch elements (all channels),
    one batch element at a time, until `seconds` elapse (or the batch ends,
    unless `wrap` cycles over it again).  Returns (modeled
    bytes processed, wall seconds, planes, cores, description)."""
    import numpy as np

    import oracle
    from wtconv_inputs import make_inputs

    orc = oracle.default()
    sub = case.with_(B=1)
    done_planes, t_total, nbytes = 0, 0.0, 0
    b = 0
    mb = modeled_bytes(sub)
    per_b = sum(mb.values())
    while True:
        inp = make_inputs(sub.with_(seed=case.seed + b % case.B))
        p = {k: inp[k].double().numpy() for k in ("base_w", "base_b", "base_scale", "wt_w", "wt_scale")}
        x, dy = inp["x"].double().numpy(), inp["dy"].double().numpy()
        t0 = time.perf_counter()
        orc.forward(x, p["base_w"], p["base_b"], p["base_scale"], p["wt_w"], p["wt_scale"], case.L)
        orc.backward_input(dy, p["base_w"], p["base_scale"], p["wt_w"], p["wt_scale"], case.L)
        orc.backward_weight(x, dy, p["base_w"], p["base_b"], p["base_scale"], p["wt_w"], p["wt_scale"], case.L)
        t_total += time.perf_counter() - t0
        nbytes += per_b
        done_planes += case.C
        b += 1
        if t_total >= seconds or (not wrap and b >= case.B) or (max_planes and done_planes >= max_planes):
            break
    desc = (f"{b} batch elements (cycling over the {case.B} of the workload) x all {case.C} channels "
            f"({done_planes} planes), forward + backward_input + backward_weight in float64")
    return nbytes, t_total, done_planes, orc.num_threads(), desc


def run_reference(args, case):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    # Calibrate one batch element, then size each step to keep the run short.
    nbytes, t1, _, cores, _ = oracle_sample(case, 0.0)
    budget = 120.0
    steps = max(1, args.steps)
    per_step_target = max(0.05, budget / (steps + args.warmup))
    n_b = max(1, min(case.B, int(per_step_target / max(t1, 1e-6))))
    sub = case.with_(B=n_b)
    for _ in range(args.warmup):
        oracle_sample(sub, 0.0, max_planes=1)
    t_sum, b_sum = 0.0, 0
    for _ in range(steps):
        nb, t, _, _, _ = oracle_sample(sub, 1e9)
        t_sum += t
        b_sum += nb
    value = b_sum / t_sum / 1e9
    ms = 1e3 * t_sum / steps
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_name(case), "sample_batch_per_step": n_b},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"{n_b} of {case.B} batch elements x all {case.C} channels per step"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------
# The CUDA path.
# --------------------------------------------------------------------------
class Workload:
    """Device buffers of one workload and its three calls (plus, with several
    ranks, the all-reduce of the weight gradients)."""

    def __init__(self, case, dev, stream, rank: int, world: int, nhwc: bool = False):
        import torch

        import memory_bound_cnn_wtconv_b200 as wt
        from wtconv_inputs import make_inputs

        self.case, self.dev, self.stream, self.world = case, dev, stream, world
        inp = make_inputs(case.with_(seed=case.seed + 7919 * rank))
        self.g = g = {k: v.to(dev) for k, v in inp.items()}
        if nhwc:  # channels-last activations (same values, NHWC storage)
            for k in ("x", "dy"):
                g[k] = g[k].contiguous(memory_format=torch.channels_last)
        L = case.L
        self.y = torch.empty_like(g["x"])
        self.dx = torch.empty_like(g["dy"])
        self.grads = grads = {k: torch.empty_like(g[k]) for k in ("base_w", "base_b", "base_scale", "wt_w", "wt_scale")}
        self.flat = torch.empty(sum(v.numel() for v in grads.values()), device=dev)
        self.ws = torch.empty(max(16, wt.workspace_bytes(g["x"].shape, case.k, L, g["x"].dtype, channels_last=nhwc)),
                              dtype=torch.uint8, device=dev)

        def fwd():
            wt.forward(g["x"], g["base_w"], g["base_b"], g["base_scale"], g["wt_w"], g["wt_scale"], L, y=self.y,
                       stream=stream)

        def bwd_in():
            wt.backward_input(g["dy"], g["base_w"], g["base_scale"], g["wt_w"], g["wt_scale"], L, dx=self.dx,
                              stream=stream)

        def bwd_w():
            wt.backward_weight(g["x"], g["dy"], g["base_w"], g["base_b"], g["base_scale"], g["wt_w"], g["wt_scale"], L,
                               grads=grads, workspace=self.ws, stream=stream)

        def bwd_fused():
            wt.backward(g["x"], g["dy"], g["base_w"], g["base_b"], g["base_scale"], g["wt_w"], g["wt_scale"], L,
                        dx=self.dx, grads=grads, workspace=self.ws, stream=stream)

        def bwd_one_pass():
            wt.backward(g["x"], g["dy"], g["base_w"], g["base_b"], g["base_scale"], g["wt_w"], g["wt_scale"], L,
                        dx=self.dx, grads=grads, workspace=self.ws, stream=stream, one_pass=True)

        self.calls = [("fwd", fwd), ("bwd_in", bwd_in), ("bwd_w", bwd_w)]
        if world > 1:
            import torch.distributed as dist
            self.calls.append(("allreduce", lambda: allreduce_weight_grads(grads, self.flat, dist)))
        self.bwd_fused = bwd_fused
        # The one-pass kernel, where the shape has a one-pass plan.
        try:
            bwd_one_pass()
            self.bwd_one_pass = bwd_one_pass
        except wt.WTConvError as e:
            if e.code != 8:  # WTCONV_ERR_UNSUPPORTED: planes split into cluster strips
                raise
            self.bwd_one_pass = None

    def time_calls(self, calls, steps: int, warmup: int, flush, clocks=None):
        """Per-call device times (ms) of `steps` timed steps after `warmup`
        untimed ones: CUDA events on the launching stream around every call,
        L2 flushed (a 256 MiB write) before every call.  Returns the lists of
        per-call times and the wall time of the timed region."""
        import torch
        for _ in range(warmup):
            for _, f in calls:
                flush.zero_()
                f()
        torch.cuda.synchronize(self.dev)
        ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in calls]
              for _ in range(steps)]
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize(self.dev)
        wall0 = time.perf_counter()
        for s in range(steps):
            for i, (_, f) in enumerate(calls):
                flush.zero_()
                ev[s][i][0].record(self.stream)
                f()
                ev[s][i][1].record(self.stream)
        torch.cuda.synchronize(self.dev)
        if self.world > 1:
            import torch.distributed as dist
            dist.barrier()
        wall = time.perf_counter() - wall0
        clk = clocks.stop() if clocks is not None else None
        times = {name: [ev[s][i][0].elapsed_time(ev[s][i][1]) for s in range(steps)] for i, (name, _) in enumerate(calls)}
        return times, wall, clk


def call_record(case, per_call_ms: dict, peak: float, nhwc: bool = False) -> dict:
    """GB/s, HBM fraction and FP32-pipe fraction of each call and of the step."""
    mb = modeled_bytes(case)
    alu_peak = SMS * FP32_LANES * 2 * MAX_SM_MHZ * 1e6 / 1e12
    step_ms = sum(per_call_ms[k] for k in mb)
    gbs = sum(mb.values()) / (step_ms * 1e-3) / 1e9
    return {
        "workload": workload_name(case, nhwc),
        "us_per_call": {k: per_call_ms[k] * 1e3 for k in mb},
        "gbs_per_call": {k: mb[k] / (per_call_ms[k] * 1e-3) / 1e9 for k in mb},
        "hbm_frac_per_call": {k: mb[k] / (per_call_ms[k] * 1e-3) / 1e9 / peak for k in mb},
        "alu_frac_per_call": {k: 2.0 * conv_fmas(case) / (per_call_ms[k] * 1e-3) / 1e12 / alu_peak for k in mb},
        "step_us": step_ms * 1e3, "step_gbs": gbs, "step_hbm_frac": gbs / peak,
        "modeled_bytes_per_step": sum(mb.values()),
    }


def median(v):
    return statistics.median(v)


def backward_record(wl, case, per_call_ms: dict, steps: int, flush, dist=None, dev=None) -> tuple:
    """The whole-backward calls beside the two passes, same protocol: the
    library's pick (wtconv_backward) and the one-pass kernel
    (wtconv_backward_one_pass).  Returns (record, kernel launches timed)."""
    calls = [("library_pick", wl.bwd_fused)]
    if wl.bwd_one_pass is not None:
        calls.append(("one_pass", wl.bwd_one_pass))
    t, _, _ = wl.time_calls(calls, steps, 3, flush)
    ms = {n: median(v) for n, v in t.items()}
    if dist is not None:
        ms = {n: max_over_ranks(v, dist, dev) for n, v in ms.items()}
    two = per_call_ms["bwd_in"] + per_call_ms["bwd_w"]
    fb_bytes = 3 * case.numel * case.esize + 2 * 4 * param_floats(case)
    rec = {
        "call": "wtconv_backward: dx and all parameter gradients (the library picks the one-pass kernel or the "
                "two passes by the planner's cost); wtconv_backward_one_pass: the one-pass kernel",
        "two_pass_us": two * 1e3,
        "library_pick_us": ms["library_pick"] * 1e3,
        "one_pass_us": ms["one_pass"] * 1e3 if "one_pass" in ms else None,
        "one_pass_modeled_bytes": fb_bytes,
        "one_pass_gbs": fb_bytes / (ms["one_pass"] * 1e-3) / 1e9 if "one_pass" in ms else None,
        "step_forward_plus_library_pick_us": (per_call_ms["fwd"] + ms["library_pick"]) * 1e3,
    }
    return rec, steps * (2 + (1 if "one_pass" in ms else 0))


def run_ours(args, case):
    import torch
    import torch.distributed as dist

    import memory_bound_cnn_wtconv_b200 as wt
    from wtconv_inputs import NAMED

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    wt.load_library()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    wl = Workload(case, dev, stream, rank, world, nhwc=args.nhwc)
    K = args.steps
    clocks = Clocks(not args.no_clocks, physical_gpu_index(local))
    times, wall, clk = wl.time_calls(wl.calls, K, args.warmup, flush, clocks)
    # Per-call medians over the K timed steps; the step is their sum.
    per_call = {name: median(v) for name, v in times.items()}
    step_ms = sum(per_call.values())
    if world > 1:
        step_ms = max_over_ranks(step_ms, dist, dev)

    mb = modeled_bytes(case)
    step_bytes = sum(mb.values())
    value = step_bytes * world / (step_ms * 1e-3) / 1e9
    peak, peak_kind = hbm_peak()

    # Dominant kernel (largest share of the step) and its roofline.
    dom = max(("fwd", "bwd_in", "bwd_w"), key=lambda n: per_call[n])
    dom_s = per_call[dom] * 1e-3
    flops = 2.0 * conv_fmas(case)
    alu_peak = SMS * FP32_LANES * 2 * MAX_SM_MHZ * 1e6 / 1e12  # TFLOP/s
    alu_achieved = flops / dom_s / 1e12
    hbm_achieved = mb[dom] / dom_s / 1e9
    t_alu, t_hbm = flops / (alu_peak * 1e12), mb[dom] / (peak * 1e9)
    kernel_names = {"fwd": "wtconv_fused_kernel (forward)", "bwd_in": "wtconv_fused_kernel (input gradient)",
                    "bwd_w": "wtconv_bwdw_partial_kernel (final step in its tail)"}
    traffic, traffic_src = measured_traffic(case.name, dom)
    if t_alu >= t_hbm:
        roof = {"bound": "alu", "achieved": alu_achieved, "peak": alu_peak, "unit": "TFLOP/s",
                "frac": alu_achieved / alu_peak, "traffic": traffic, "traffic_source": traffic_src,
                "kernel": kernel_names[dom],
                "peak_source": "148 SMs x 128 FP32 FMA lanes x 2 x 1965 MHz (unit counts x max clock)",
                "flops_per_launch": flops, "hbm_frac": hbm_achieved / peak, "bytes_per_launch": mb[dom]}
    else:
        roof = {"bound": "hbm", "achieved": hbm_achieved, "peak": peak, "unit": "GB/s", "frac": hbm_achieved / peak,
                "traffic": traffic, "traffic_source": traffic_src, "kernel": kernel_names[dom],
                "peak_source": peak_kind,
                "bytes_per_launch": mb[dom]}

    rec = call_record(case, per_call, peak, args.nhwc)
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if case.dtype == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": workload_name(case, args.nhwc), "global_batch": case.B * world,
                   "parallelism": f"dp{world}", "l2": "flushed before every call (256 MiB write)",
                   "timing": f"median over the {K} timed steps of each call's CUDA-event time; step = their sum",
                   "modeled_bytes_per_step": step_bytes},
        "hbm_frac_of_peak": value / world / peak, "hbm_peak_gbs": peak, "hbm_peak_source": peak_kind,
        "frac_of_8tbs": value / world / 8000.0,
        "us_per_call": {k: v * 1e3 for k, v in per_call.items()},
        "gbs_per_call": rec["gbs_per_call"],
        "roofline": roof,
        "alu_frac_per_call": rec["alu_frac_per_call"],
        # Our kernels in the timed region: forward, input gradient, weight
        # gradient (its final step runs in the same launch) per step.
        "gpu_launches": K * 3, "wall_s_timed_region": wall,
    }
    if clk is not None:
        line["clocks"] = clk

    if not args.no_e2e:
        line["e2e"] = e2e(args, case, wl.g, wl.grads, wl.ws, dev, world)
    if world > 1:
        dist.barrier()
    # The whole-backward calls (library pick, one-pass kernel), timed after
    # the step with the same protocol; reported beside the three-call step,
    # not in it.
    KF = min(K, 500)
    line["fused_backward"], n_launch = backward_record(wl, case, per_call, KF, flush,
                                                       dist if world > 1 else None, dev)
    line["gpu_launches"] += n_launch
    # The other WTConvNeXt stage shapes, same protocol, one GPU.
    if world == 1 and not args.no_other_workloads and not args.nhwc:
        other = {}
        for name in ("stage1", "stage2", "train_bf16", "stage1_nhwc"):
            if name == case.name:
                other[name] = dict(rec, fused_backward=line["fused_backward"])
                continue
            nhwc = name.endswith("_nhwc")
            wcase = NAMED[name[:-len("_nhwc")] if nhwc else name]
            del_wl = Workload(wcase, dev, stream, 0, 1, nhwc=nhwc)
            t2, _, _ = del_wl.time_calls(del_wl.calls, K, args.warmup, flush)
            pc2 = {n: median(v) for n, v in t2.items()}
            other[name] = call_record(wcase, pc2, peak, nhwc)
            other[name]["fused_backward"], n_launch = backward_record(del_wl, wcase, pc2, KF, flush)
            line["gpu_launches"] += K * 3 + n_launch
            del del_wl
            torch.cuda.empty_cache()
        line["workloads"] = other
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        nb, t, planes, cores, desc = oracle_sample(case, args.cpu_seconds, wrap=True)
        line["cpu_baseline"] = {"value": nb / t / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
                                "sample": desc, "seconds": t}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def e2e(args, case, g, grads, ws, dev, world):
    """Same metric through the public API with host buffers: every step copies
    x and dy from pinned host memory to the device, runs the three calls (and,
    with several ranks, the gradient all-reduce), and copies y, dx and the
    gradients back.  Steps are pipelined over three streams (inputs, compute,
    results) with two device buffer sets, so one step's copies in and out
    overlap the neighbouring steps' compute; events keep every buffer from
    being overwritten before its last reader is done."""
    import torch
    import torch.distributed as dist

    import memory_bound_cnn_wtconv_b200 as wt

    L = case.L
    xh = g["x"].cpu().pin_memory()
    dyh = g["dy"].cpu().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    dxh = torch.empty_like(dyh).pin_memory()
    gh = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in grads.items()}
    bufs = [dict(x=torch.empty_like(g["x"]), dy=torch.empty_like(g["dy"]), y=torch.empty_like(g["x"]),
                 dx=torch.empty_like(g["dy"]), grads={k: torch.empty_like(v) for k, v in grads.items()})
            for _ in range(2)]
    flat = torch.empty(sum(v.numel() for v in grads.values()), device=dev)
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    done = {"in": [None, None], "comp": [None, None], "out": [None, None]}

    def mark(kind, b, strm):
        e = torch.cuda.Event()
        e.record(strm)
        done[kind][b] = e

    def step(i):
        b = i % 2
        d = bufs[b]
        with torch.cuda.stream(s_in):
            if done["comp"][b] is not None:
                s_in.wait_event(done["comp"][b])  # step i-2 no longer reads x, dy of this set
            d["x"].copy_(xh, non_blocking=True)
            d["dy"].copy_(dyh, non_blocking=True)
            mark("in", b, s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(done["in"][b])
            if done["out"][b] is not None:
                s_comp.wait_event(done["out"][b])  # step i-2's results are on the host
            wt.forward(d["x"], g["base_w"], g["base_b"], g["base_scale"], g["wt_w"], g["wt_scale"], L, y=d["y"],
                       stream=s_comp)
            wt.backward_input(d["dy"], g["base_w"], g["base_scale"], g["wt_w"], g["wt_scale"], L, dx=d["dx"],
                              stream=s_comp)
            wt.backward_weight(d["x"], d["dy"], g["base_w"], g["base_b"], g["base_scale"], g["wt_w"], g["wt_scale"],
                               L, grads=d["grads"], workspace=ws, stream=s_comp)
            if world > 1:
                allreduce_weight_grads(d["grads"], flat, dist)
            mark("comp", b, s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(done["comp"][b])
            yh.copy_(d["y"], non_blocking=True)
            dxh.copy_(d["dx"], non_blocking=True)
            for k in gh:
                gh[k].copy_(d["grads"][k], non_blocking=True)
            mark("out", b, s_out)

    for i in range(3):
        step(i)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    K = args.e2e_steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(K):
        step(i)
    e1.record(s_out)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / K
    if world > 1:
        ms = max_over_ranks(ms, dist, dev)
    step_bytes = sum(modeled_bytes(case).values())
    h2d = xh.numel() * xh.element_size() + dyh.numel() * dyh.element_size()
    d2h = yh.numel() * yh.element_size() + dxh.numel() * dxh.element_size() + sum(
        v.numel() * v.element_size() for v in gh.values())
    return {"value": step_bytes * world / (ms * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": K,
            "pipelined": "3 streams (copy in / compute / copy out), 2 device buffer sets"}


# --------------------------------------------------------------------------
# Comparators: the same layer as separate PyTorch library ops with every
# intermediate in memory (the unfused formulation the pages measure the
# fused one against), and the plain depthwise conv the layer extends.
# Context numbers only, printed by --compare; never the product path.
# --------------------------------------------------------------------------
def haar_filters(C: int, dtype, device):
    """The four orthonormal 2x2 Haar analysis filters (LL, LH, HL, HH) for
    every channel, as grouped-conv weights [4C, 1, 2, 2]."""
    import torch
    f = torch.tensor([[[1, 1], [1, 1]], [[1, 1], [-1, -1]], [[1, -1], [1, -1]], [[1, -1], [-1, 1]]],
                     dtype=dtype, device=device) * 0.5
    return f.unsqueeze(1).repeat(C, 1, 1, 1)


def unfused_wtconv(x, base_w, base_b, base_scale, wt_w, wt_scale, L: int):
    """The layer level by level with PyTorch ops: Haar analysis as a stride-2
    grouped conv, one grouped conv per level for the 4C subbands, scaling,
    and the synthesis as a stride-2 grouped transposed conv adding each
    coarser level into the next finer LL.  Differentiable."""
    import torch
    import torch.nn.functional as F
    B, C, H, W = x.shape
    k = base_w.shape[-1]
    p = k // 2
    dt = x.dtype
    y = F.conv2d(x, base_w.to(dt).unsqueeze(1), base_b.to(dt), padding=p, groups=C)
    y = y * base_scale.to(dt).view(1, C, 1, 1)
    if L == 0:
        return y
    filt = haar_filters(C, dt, x.device)
    ll, shat = x, []
    for l in range(L):
        s = F.conv2d(ll, filt, stride=2, groups=C)
        h, w = s.shape[-2:]
        z = F.conv2d(s, wt_w[l].to(dt).reshape(4 * C, 1, k, k), padding=p, groups=4 * C)
        shat.append(z * wt_scale[l].to(dt).reshape(1, 4 * C, 1, 1))
        ll = s.view(B, C, 4, h, w)[:, :, 0]
    zc = None
    for l in range(L - 1, -1, -1):
        z = shat[l]
        if zc is not None:
            h, w = z.shape[-2:]
            z4 = z.view(B, C, 4, h, w)
            z = torch.cat([z4[:, :, :1] + zc.unsqueeze(2), z4[:, :, 1:]], dim=2).view(B, 4 * C, h, w)
        zc = F.conv_transpose2d(z, filt, stride=2, groups=C)
    return y + zc


def depthwise_conv(x, base_w, base_b):
    """The plain depthwise k x k conv (cuDNN through PyTorch)."""
    import torch.nn.functional as F
    C, k = x.shape[1], base_w.shape[-1]
    return F.conv2d(x, base_w.to(x.dtype).unsqueeze(1), base_b.to(x.dtype), padding=k // 2, groups=C)


def run_compare(args, case):
    """Forward and forward+backward time and the peak memory of one training
    step: the fused library (autograd function), the unfused PyTorch layer,
    and the plain depthwise conv; one JSON line each."""
    import torch

    import memory_bound_cnn_wtconv_b200 as wt
    from wtconv_inputs import make_inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    inp = make_inputs(case)
    g = {k: v.to(dev) for k, v in inp.items()}
    params = {k: g[k].clone().requires_grad_(True) for k in ("base_w", "base_b", "base_scale", "wt_w", "wt_scale")}
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    impls = {
        "fused (this library)": lambda x: wt.wtconv(x, params["base_w"], params["base_b"], params["base_scale"],
                                                    params["wt_w"], params["wt_scale"], case.L),
        "unfused PyTorch ops": lambda x: unfused_wtconv(x, params["base_w"], params["base_b"], params["base_scale"],
                                                        params["wt_w"], params["wt_scale"], case.L),
        "depthwise conv only (PyTorch)": lambda x: depthwise_conv(x, params["base_w"], params["base_b"]),
    }

    def timed(fn, reps):
        ts = []
        for _ in range(reps):
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e3)
        return statistics.median(ts)

    if args.compare_only:
        impls = {k: v for k, v in impls.items() if k.startswith(args.compare_only)}
    for name, f in impls.items():
        x = g["x"].clone().requires_grad_(True)
        dy = g["dy"]
        if args.profile_one_forward:
            # For an ncu run with --profile-from-start off: warm up, then
            # exactly one forward between profiler start and stop.
            for _ in range(3):
                f(x).backward(dy)
            torch.cuda.synchronize()
            flush.fill_(1)
            torch.cuda.synchronize()
            torch.cuda.profiler.start()
            with torch.no_grad():
                f(x)
            torch.cuda.synchronize()
            torch.cuda.profiler.stop()
            continue

        def fwd():
            with torch.no_grad():
                f(x)

        def step():
            y = f(x)
            y.backward(dy)

        for _ in range(max(3, args.warmup)):
            step()
        torch.cuda.synchronize()
        t_f = timed(fwd, args.steps)
        t_s = timed(step, args.steps)
        x.grad = None
        for v in params.values():
            v.grad = None
        torch.cuda.synchronize()
        base = torch.cuda.memory_allocated(dev)
        torch.cuda.reset_peak_memory_stats(dev)
        step()
        torch.cuda.synchronize()
        peak = torch.cuda.max_memory_allocated(dev) - base
        print(json.dumps({"impl": "compare", "what": name, "config": {"workload": workload_name(case)},
                          "us_forward": t_f, "us_forward_backward": t_s, "peak_extra_bytes_train_step": peak,
                          "dtype": case.dtype, "l2": "flushed before every timed call"}), flush=True)
        x.grad = None
        for v in params.values():
            v.grad = None
    return 0


def run_sweep(args):
    """Per-call device time (CUDA events, L2 flushed before every call) of the
    forward, input gradient and weight gradient at each sweep point; one JSON
    line per point, then a summary line.  One GPU."""
    import torch

    import memory_bound_cnn_wtconv_b200 as wt
    from wtconv_inputs import make_inputs, sweep_cases

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    wt.load_library()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    cases = sweep_cases()
    if args.sweep_points:
        if ":" in args.sweep_points:
            a, b = (int(v) if v else None for v in args.sweep_points.split(":"))
            cases = cases[a:b]
        else:
            cases = [cases[int(args.sweep_points)]]
    peak, peak_kind = hbm_peak()
    alu_peak = 148 * 128 * 2 * 1965e6
    rows = []
    for case in cases:
        g = {k: v.to(dev) for k, v in make_inputs(case).items()}
        L = case.L
        y, dx = torch.empty_like(g["x"]), torch.empty_like(g["dy"])
        grads = {k: torch.empty_like(g[k]) for k in ("base_w", "base_b", "base_scale", "wt_w", "wt_scale")}
        ws = torch.empty(max(16, wt.workspace_bytes(g["x"].shape, case.k, L, g["x"].dtype)), dtype=torch.uint8,
                         device=dev)
        calls = {
            "fwd": lambda: wt.forward(g["x"], g["base_w"], g["base_b"], g["base_scale"], g["wt_w"], g["wt_scale"], L,
                                      y=y, stream=stream),
            "bwd_in": lambda: wt.backward_input(g["dy"], g["base_w"], g["base_scale"], g["wt_w"], g["wt_scale"], L,
                                                dx=dx, stream=stream),
            "bwd_w": lambda: wt.backward_weight(g["x"], g["dy"], g["base_w"], g["base_b"], g["base_scale"], g["wt_w"],
                                                g["wt_scale"], L, grads=grads, workspace=ws, stream=stream),
        }
        def one_pass():
            wt.backward(g["x"], g["dy"], g["base_w"], g["base_b"], g["base_scale"], g["wt_w"], g["wt_scale"], L,
                        dx=dx, grads=grads, workspace=ws, stream=stream, one_pass=True)
        try:  # the one-pass backward kernel, timed beside the step where the shape has a plan for it
            one_pass()
            calls["one_pass_bwd"] = one_pass
        except wt.WTConvError as e:
            if e.code != 8:
                raise
        us = {}
        for name, f in calls.items():
            for _ in range(3):
                f()
            ev = []
            for _ in range(args.sweep_steps):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                f()
                e1.record(stream)
                ev.append((e0, e1))
            torch.cuda.synchronize(dev)
            us[name] = sorted(a.elapsed_time(b) for a, b in ev)[len(ev) // 2] * 1e3
        mb = modeled_bytes(case)
        one_pass_us = us.pop("one_pass_bwd", None)
        step_us = sum(us.values())
        gbs = sum(mb.values()) / (step_us * 1e-6) / 1e9
        alu = 3 * 2 * conv_fmas(case) / (step_us * 1e-6) / alu_peak
        row = {"sweep_point": case.name, "B": case.B, "C": case.C, "H": case.H, "k": case.k, "L": case.L,
               "us": {k: round(v, 1) for k, v in us.items()}, "step_us": round(step_us, 1),
               "gbs": round(gbs, 1), "hbm_frac": round(gbs / peak, 4), "alu_frac": round(alu, 4),
               "one_pass_bwd_us": None if one_pass_us is None else round(one_pass_us, 1)}
        rows.append(row)
        print(json.dumps(row), flush=True)
        del g, y, dx, grads, ws
        torch.cuda.empty_cache()
    gb = sorted(r["gbs"] for r in rows)
    print(json.dumps({"sweep_points": len(rows), "gbs_median": gb[len(gb) // 2], "gbs_min": gb[0], "gbs_max": gb[-1],
                      "hbm_peak_gbs": peak, "hbm_peak_source": peak_kind, "timing": "median of per-call CUDA events, "
                      "L2 flushed before every call", "data": "synthetic"}))
    return 0


def relaunch(args) -> int:
    """`--gpus N` (N > 1) outside a torch.distributed launch: run this script
    again as N ranks on this node (one per GPU) through torch.distributed.run,
    rendezvous on 127.0.0.1, and return its exit status."""
    import signal
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *sys.argv[1:]]
    proc = subprocess.Popen(cmd, start_new_session=True)
    try:
        return proc.wait(timeout=1800)
    except subprocess.TimeoutExpired:
        os.killpg(proc.pid, signal.SIGTERM)
        try:
            proc.wait(timeout=60)
        except subprocess.TimeoutExpired:
            os.killpg(proc.pid, signal.SIGKILL)
        return 124


def run_dist_check(args) -> int:
    """The multi-rank path without kernels (gloo on the CPU): each rank fills
    its weight gradients with rank-dependent values, sums them over the ranks
    with the bench's all-reduce, checks the sums, and reports the slowest
    rank's time.  Rank 0 prints one JSON line."""
    import torch
    import torch.distributed as dist

    world, rank, _ = dist_env()
    if world > 1:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    case = __import__("wtconv_inputs").TINY
    shapes = {"base_w": (case.C, case.k, case.k), "base_b": (case.C,), "base_scale": (case.C,),
              "wt_w": (case.L, case.C, 4, case.k, case.k), "wt_scale": (case.L, case.C, 4)}
    grads = {k: torch.full(v, float(rank + 1)) for k, v in shapes.items()}
    flat = torch.empty(sum(v.numel() for v in grads.values()))
    t0 = time.perf_counter()
    for _ in range(max(1, args.steps)):
        for v in grads.values():
            v.fill_(float(rank + 1))
        if world > 1:
            allreduce_weight_grads(grads, flat, dist)
    t = time.perf_counter() - t0
    ok = all(bool(torch.all(v == world * (world + 1) / 2)) for v in grads.values())
    if world > 1:
        t = max_over_ranks(t, dist, torch.device("cpu"))
        okt = torch.tensor([1 if ok else 0])
        dist.all_reduce(okt, op=dist.ReduceOp.MIN)
        ok = bool(okt.item())
    if rank == 0:
        print(json.dumps({"impl": "dist-check", "n_gpus": world, "steps": args.steps, "backend": "gloo",
                          "allreduce_sum_ok": ok, "s_max_over_ranks": t}), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0 if ok else 1


def main():
    args = parse()
    env_world = os.environ.get("WORLD_SIZE")
    if env_world is None and args.gpus > 1:
        return relaunch(args)
    if env_world is not None and int(env_world) != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={env_world}; launch one rank per GPU", file=sys.stderr)
        return 2
    if args.dist_check:
        return run_dist_check(args)
    if args.sweep:
        return run_sweep(args)
    from wtconv_inputs import NAMED, sweep_cases
    sweep = {c.name: c for c in sweep_cases()}
    if args.workload in NAMED:
        case = NAMED[args.workload]
    elif args.workload in sweep or args.workload.startswith("sweep"):
        # A point of the 128-point shape sweep, by full name or index ("sweep031").
        by_index = {c.name[:8]: c for c in sweep.values()}
        case = sweep.get(args.workload) or by_index.get(args.workload[:8])
        if case is None:
            raise SystemExit(f"unknown sweep point {args.workload}")
    else:
        raise SystemExit(f"unknown workload {args.workload}; choose from {sorted(NAMED)} or sweepNNN")
    if case.name == "tiny":
        case = case.with_(calls=("fwd", "bwd_in", "bwd_w"))
    if args.impl == "reference":
        return run_reference(args, case)
    if args.compare:
        return run_compare(args, case)
    return run_ours(args, case)


if __name__ == "__main__":
    sys.exit(main())
