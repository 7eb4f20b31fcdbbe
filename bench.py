#!/usr/bin/env python
"""Benchmark of the displaced-patch block step; rank 0 prints one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one ``dp_block_step`` of the workload (default: the SDXL 1024 px
top-resolution ResBlock, latent 1x320x128x128, P = 4 bands) in displaced mode,
on synthetic inputs already resident in HBM.  Each step is timed with CUDA
events recorded on the launching stream just before and after it; L2 is
flushed (a 256 MiB write) between steps, outside the timed events.  A second
pass with an event before every kernel (``dp_block_step_timed``) gives the
per-kernel breakdown and the roofline of the dominant kernel.
With N > 1 (torchrun) every rank runs an independent replica on its own GPU:
the path has no data exchange on one GPU per image, so there is no
collective; the time is the max over ranks.

``--impl reference`` times the CPU oracle instead (the only reference this
method has), on the host cores, on a row crop of the same block sized so the
whole run stays within a few minutes.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "displaced U-Net block step latency & TFLOP/s; GroupNorm GB/s; % of roofline"
FLUSH_BYTES = 256 << 20
# GroupNorm statistics of the displaced steps (--gn-stats): the method's
# corrected statistics (default) or one of its ablation alternatives
GN_STATS_NAMES = ["corrected", "local", "stale", "sync"]
GN_STATS = 0


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def kernel_source_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "displaced_patch_parallelism_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def load_traffic(key, src_hash):
    """DRAM bytes per launch from a committed ncu summary, if it matches the current source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(key)
    if not e or e.get("source_hash") != src_hash:
        return None
    return e.get("bytes_per_launch")


class ClockSampler:
    """Samples SM clock and throttle reasons while the timed region runs."""

    REASONS = {0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index):
        self.dev = device_index
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def start(self):
        if self.ok:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread:
            self._stop.set()
            self._thread.join()
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(x, dist, device):
    """The largest of every rank's x (the job's time is the slowest replica's)."""
    if dist is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world_size, flops_per_step, steps, total_ms):
    """Whole-job throughput: every replica runs `steps` steps of `flops_per_step`."""
    return world_size * flops_per_step * steps / (total_ms * 1e-3) / 1e12


def block_kind(B, wl):
    return {"gn_conv": B.GN_CONV, "resblock": B.RESBLOCK, "attn": B.ATTN,
            "unet_mini": B.UNET_MINI, "transformer": B.TRANSFORMER}[wl.kind]


def wl_context(wl):
    """(ctx_len, ctx_dim, ff_inner) of a transformer workload, else None."""
    return (wl.ctx_len, wl.ctx_dim, wl.ff_inner) if wl.kind == "transformer" else None


def oracle_context(wl):
    """A transformer workload's text context for the oracle (fp64), else None."""
    from displaced_patch_parallelism_b200 import synth
    return synth.context(wl).double().numpy() if wl.kind == "transformer" else None


def block_desc(B, wl, H=None):
    d = B.dp_block_desc_init(block_kind(B, wl), H or wl.H, wl.W, wl.C, wl.cout, wl.G, wl.P,
                             wl.heads, B.BF16 if wl.dtype == "bf16" else B.FP32, wl.silu,
                             wl.eps, 1.0)
    if wl_context(wl):
        B.dp_block_desc_set_context(d, *wl_context(wl))
    B.dp_block_desc_set_gn_stats(d, GN_STATS)
    return d


def launch_plan(B, wl, mode):
    """(kernel, algorithmic flops, algorithmic bytes) of every launch of one block step,
    as the library reports them from the step's own code path."""
    d = block_desc(B, wl)
    return [B.dp_block_launch_info(d, mode, i) for i in range(B.dp_block_launch_count(d))]


def cpu_baseline_ours(wl, seconds):
    """The oracle, as it stands, timed on this host: full displaced steps until `seconds` pass."""
    from displaced_patch_parallelism_b200 import synth
    from oracle import dp_oracle as O
    wts = {n: v.double().numpy() for n, v in synth.make_weights(wl).items()}
    xs = synth.InputStream(wl)
    ctx = oracle_context(wl)
    st = {}
    O.block_step(wl.kind, st, xs.x(0)[0], wts, wl.P, wl.G, wl.eps, 1.0, synth.SYNC, wl.dtype,
                 heads=wl.heads, silu=wl.silu, ctx=ctx)
    x1 = xs.x(1)[0]
    reps, t0 = 0, time.perf_counter()
    while True:
        O.block_step(wl.kind, st, x1, wts, wl.P, wl.G, wl.eps, 1.0, synth.DISPLACED, wl.dtype,
                     heads=wl.heads, silu=wl.silu, gn_stats=GN_STATS, ctx=ctx)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return reps, el


def wl_flops(wl, H=None):
    from displaced_patch_parallelism_b200 import binding as B
    return B.dp_block_flops(block_desc(B, wl, H))


def run_reference(args, wl):
    """The CPU oracle on the host cores: each step a displaced step of a row crop of the block."""
    import dataclasses

    from displaced_patch_parallelism_b200 import synth
    from oracle import dp_oracle as O
    budget = 150.0
    cores = len(os.sched_getaffinity(0))
    ctx = oracle_context(wl)

    def crop(rows_per_band):
        return dataclasses.replace(wl, H=wl.P * rows_per_band)

    def one_step_time(w):
        wts = {n: v.double().numpy() for n, v in synth.make_weights(w).items()}
        xs = synth.InputStream(w)
        st = {}
        O.block_step(w.kind, st, xs.x(0)[0], wts, w.P, w.G, w.eps, 1.0, synth.SYNC, w.dtype,
                     heads=w.heads, silu=w.silu, ctx=ctx)
        t0 = time.perf_counter()
        O.block_step(w.kind, st, xs.x(1)[0], wts, w.P, w.G, w.eps, 1.0, synth.DISPLACED, w.dtype,
                     heads=w.heads, silu=w.silu, gn_stats=GN_STATS, ctx=ctx)
        return time.perf_counter() - t0, wts, st, xs

    hb = wl.H // wl.P
    if wl.kind in ("attn", "transformer"):
        rows = hb  # attention blocks need whole 128-token tiles: keep the full image
    else:
        t_small, *_ = one_step_time(crop(2))
        per_row = t_small / (2 * wl.P)
        fit = int((budget / max(1, args.steps + args.warmup)) / max(per_row, 1e-6) / wl.P)
        rows = max(2, min(hb, fit))
    w = crop(rows)
    _, wts, st, xs = one_step_time(w)
    x = xs.x(2)[0]
    for _ in range(args.warmup):
        O.block_step(w.kind, st, x, wts, w.P, w.G, w.eps, 1.0, synth.DISPLACED, w.dtype,
                     heads=w.heads, silu=w.silu, gn_stats=GN_STATS, ctx=ctx)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        O.block_step(w.kind, st, x, wts, w.P, w.G, w.eps, 1.0, synth.DISPLACED, w.dtype,
                     heads=w.heads, silu=w.silu, gn_stats=GN_STATS, ctx=ctx)
    el = time.perf_counter() - t0
    flops = wl_flops(wl, w.H)
    value = flops * args.steps / el / 1e12
    sample = (f"displaced step of the {wl.name} block on a {w.C}x{w.H}x{w.W} row crop "
              f"({rows} rows per band, {flops / 1e9:.2f} GFLOP per step)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "shape_nchw": [1, wl.C, wl.H, wl.W], "P": wl.P,
                       "mode": "displaced", "gn_stats": GN_STATS_NAMES[GN_STATS], "sample": sample},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, wl):
    import torch

    from displaced_patch_parallelism_b200 import binding as B
    from displaced_patch_parallelism_b200 import synth
    from displaced_patch_parallelism_b200.weights import block_weights

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dist = None
    if ws > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    wts = synth.make_weights(wl)
    dw = block_weights(wl.kind, wts, tdt, dev)
    if wl.kind == "transformer":     # the step's text context is the last pointer
        dw.append(synth.context(wl).to(tdt).to(dev))
    blk = B.Block(block_kind(B, wl), wl.H, wl.W, wl.C, wl.cout, wl.G, wl.P, wl.heads,
                  B.BF16 if wl.dtype == "bf16" else B.FP32, wl.silu, wl.eps, 1.0, device=dev,
                  gn_stats=GN_STATS, context=wl_context(wl))
    xs = synth.InputStream(wl)
    pool = 4
    host_x = [synth.nchw_to_nhwc(xs.x(k)).to(tdt).pin_memory() for k in range(pool)]
    dev_x = [h.to(dev) for h in host_x]
    Ho, Wo = (wl.H // 4, wl.W // 4) if wl.kind == "unet_mini" else (wl.H, wl.W)
    out = torch.empty(Ho, Wo, wl.cout, dtype=tdt, device=dev)
    host_out = torch.empty(out.shape, dtype=tdt).pin_memory()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    n_launch = blk.launches
    plan = launch_plan(B, wl, B.DISPLACED)
    assert len(plan) == n_launch
    roles = [r for r, _, _ in plan]

    warm = max(args.warmup, wl.warmup + 1)
    for i in range(warm):
        blk.step(dev_x[i % pool], out, dw, B.dp_mode_for_step(i, wl.warmup))
    torch.cuda.synchronize()

    # Timed region: one event before and one after each step, so that the
    # kernels of a step follow one another as they do in use (dependent
    # launches overlap a kernel's set-up with its predecessor).
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for e in ev0 + ev1:          # torch creates the CUDA event on its first record
        e.record()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    wall0 = time.perf_counter()
    for k in range(args.steps):
        flush.zero_()
        ev0[k].record()
        blk.step(dev_x[k % pool], out, dw, B.DISPLACED)
        ev1[k].record()
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    clocks = sampler.stop()
    if dist:
        dist.barrier()
    step_ms = [ev0[k].elapsed_time(ev1[k]) for k in range(args.steps)]
    total_ms = sum(step_ms)

    # Per-kernel breakdown: a separate pass with an event before every launch
    # (dp_block_step_timed); those events keep kernels from overlapping, so the
    # per-kernel times add up to a little more than the step above.
    n_bd = min(args.steps, 50)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(n_launch + 1)]
              for _ in range(n_bd)]
    for row in events:
        for e in row:
            e.record()
    torch.cuda.synchronize()
    for k in range(n_bd):
        flush.zero_()
        blk.step_timed(dev_x[k % pool], out, dw, B.DISPLACED, events[k])
    torch.cuda.synchronize()
    per_launch = [[events[k][i].elapsed_time(events[k][i + 1]) for i in range(n_launch)]
                  for k in range(n_bd)]
    total_ms = max_over_ranks(total_ms, dist, dev)

    # end-to-end: every step copies its input from pinned host memory, runs the
    # block step and copies its result back to pinned host memory.  The copies
    # run on their own streams (the copy engines), so step k+1's input and step
    # k's result move while a neighbouring step computes; the L2 flush stays in
    # front of every step's compute.  Timed on the device from the first copy
    # to the last.
    s_comp, s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    xin = [torch.empty_like(dev_x[0]) for _ in range(2)]
    outb = [torch.empty_like(out) for _ in range(2)]
    host_o = [host_out, torch.empty_like(host_out).pin_memory()]
    ev_in = [torch.cuda.Event() for _ in range(args.steps)]
    ev_comp = [torch.cuda.Event() for _ in range(args.steps)]
    ev_out = [torch.cuda.Event() for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t_start.record(s_comp)
    s_in.wait_event(t_start)
    for k in range(args.steps):
        b = k & 1
        if k >= 2:
            s_in.wait_event(ev_comp[k - 2])      # step k-2 has read xin[b]
        with torch.cuda.stream(s_in):
            xin[b].copy_(host_x[k % pool], non_blocking=True)
            ev_in[k].record(s_in)
        with torch.cuda.stream(s_comp):
            flush.zero_()
            s_comp.wait_event(ev_in[k])
            if k >= 2:
                s_comp.wait_event(ev_out[k - 2])  # outb[b] has reached the host
            blk.step(xin[b], outb[b], dw, B.DISPLACED)
            ev_comp[k].record(s_comp)
        s_out.wait_event(ev_comp[k])
        with torch.cuda.stream(s_out):
            host_o[b].copy_(outb[b], non_blocking=True)
            ev_out[k].record(s_out)
    s_comp.wait_event(ev_out[args.steps - 1])
    t_end.record(s_comp)
    torch.cuda.synchronize()
    e2e_ms = t_start.elapsed_time(t_end)
    e2e_ms = max_over_ranks(e2e_ms, dist, dev)
    if dist:
        dist.barrier()
    status = B.dp_device_status()

    flops = blk.flops
    value = job_tflops(ws, flops, args.steps, total_ms)
    e2e_value = job_tflops(ws, flops, args.steps, e2e_ms)

    # per-kernel roles: mean duration, share, roofline of the dominant one
    work = [(f, b) for _, f, b in plan]
    peaks = load_peaks()
    role_ms, role_n = {}, {}
    for k in range(n_bd):
        for i, r in enumerate(roles):
            role_ms[r] = role_ms.get(r, 0.0) + per_launch[k][i]
            role_n[r] = role_n.get(r, 0) + 1
    kernels = {}
    for r in role_ms:
        idx = [i for i, rr in enumerate(roles) if rr == r]
        fl = sum(work[i][0] for i in idx) / len(idx)
        by = sum(work[i][1] for i in idx) / len(idx)
        avg_us = role_ms[r] / role_n[r] * 1e3
        kernels[r] = {"launches": role_n[r], "avg_us": round(avg_us, 2),
                      "share": round(role_ms[r] / sum(role_ms.values()), 4),
                      "tflops": round(fl / (avg_us * 1e-6) / 1e12, 1) if fl else None,
                      "gbs": round(by / (avg_us * 1e-6) / 1e9, 1)}
    dominant = max(role_ms, key=lambda r: role_ms[r])
    dk = kernels[dominant]
    src = {"conv": ["dp_gemm.cu"], "linear": ["dp_gemm.cu"], "attn": ["dp_attn.cu"],
           "gn_stats": ["dp_gn.cu"], "gn_apply": ["dp_gn.cu"], "gn_fused": ["dp_gn.cu"],
           "gn_cluster": ["dp_gn.cu"],
           "copy": ["dp_refresh.cu"], "conv_small": ["dp_conv_small.cu"], "splitk_finish": ["dp_gemm.cu"]}[dominant]
    traffic = load_traffic(f"{dominant}:{wl.name}", kernel_source_hash(src))
    if dk["tflops"]:
        roof = {"bound": "tensor", "achieved": dk["tflops"], "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": round(dk["tflops"] / peaks["bf16_tflops"], 4),
                "traffic": traffic, "kernel": dominant,
                "peak_source": f"{peaks['source']} bf16 burst",
                "frac_of_sustained": round(dk["tflops"] / peaks["bf16_tflops_sustained"], 4)
                if peaks.get("bf16_tflops_sustained") else None}
    else:
        roof = {"bound": "hbm", "achieved": dk["gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(dk["gbs"] / peaks["hbm_gbs"], 4), "traffic": traffic,
                "kernel": dominant, "peak_source": f"{peaks['source']} copy"}
    gn_ms = sum(v for r, v in role_ms.items() if r.startswith("gn"))
    gn_bytes = sum(work[i][1] for i, r in enumerate(roles) if r.startswith("gn")) * n_bd
    gn = {"achieved_gbs": round(gn_bytes / (gn_ms * 1e-3) / 1e9, 1) if gn_ms else None,
          "peak": peaks["hbm_gbs"],
          "bytes_model": "single pass: read x + write y; two passes: stats read x, apply read x + write y"}
    if gn["achieved_gbs"]:
        gn["frac"] = round(gn["achieved_gbs"] / peaks["hbm_gbs"], 4)

    line = {"metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype,
            "data": "synthetic",
            "config": {"workload": wl.name, "shape_nchw": [1, wl.C, wl.H, wl.W], "P": wl.P,
                       "mode": "displaced", "gn_stats": GN_STATS_NAMES[GN_STATS],
                       "l2": "flushed between steps (256 MiB write, untimed)",
                       "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU"},
            "roofline": roof, "kernels": kernels, "groupnorm": gn,
            "e2e": {"value": round(e2e_value, 3), "unit": "TFLOP/s",
                    "copies": "input and result copies on their own streams, overlapping "
                              "neighbouring steps; L2 flushed before every step's compute",
                    "h2d_bytes_per_step": dev_x[0].numel() * dev_x[0].element_size(),
                    "d2h_bytes_per_step": out.numel() * out.element_size()},
            "gpu_launches": n_launch * args.steps, "clocks": clocks,
            "wall_s_timed_region": round(wall, 4), "device_status": status}
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        reps, el = cpu_baseline_ours(wl, args.cpu_seconds)
        line["cpu_baseline"] = {"value": round(wl_flops(wl) * reps / el / 1e12, 6), "unit": "TFLOP/s",
                                "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
                                "sample": f"{reps} full displaced steps of {wl.name} in {el:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="resblock_320x128x128")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--gn-stats", choices=GN_STATS_NAMES, default="corrected",
                    help="GroupNorm statistics of the displaced steps")
    args = ap.parse_args()
    global GN_STATS
    GN_STATS = GN_STATS_NAMES.index(args.gn_stats)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    from displaced_patch_parallelism_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        _, rank, _ = dist_env()
        if rank == 0:
            run_reference(args, wl)
        return
    run_ours(args, wl)


if __name__ == "__main__":
    main()
