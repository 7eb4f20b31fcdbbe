#!/usr/bin/env python
"""Benchmark of the displaced-patch block step; rank 0 prints one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one ``dp_block_step`` of the workload in displaced mode, on
synthetic inputs already resident in HBM.  The default workload is the largest
single-GPU one: the 3840x3840-shaped GroupNorm + SiLU + 3x3 conv block, latent
1x320x480x480, P = 8 bands of 60 rows.  Each step is timed with CUDA events
recorded on the launching stream just before and after it.  Between steps L2
is flushed (a 256 MiB write, then a 256 MiB read that writes its dirty lines back,
both outside the timed events) unless the step's input
alone is larger than L2, in which case the inputs themselves evict it.  A
second pass with an event before every kernel (``dp_block_step_timed``) gives
the per-kernel breakdown and the roofline of the dominant kernel.  The other
workloads are then timed the same way (device time and breakdown, no
end-to-end pass) and reported under ``workloads``.
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


class L2Flush:
    """Empties L2 between timed steps, outside the timed events: a 256 MiB write (evicting
    everything), then a 256 MiB read of a second buffer, which writes the first buffer's dirty
    lines back and leaves L2 holding clean lines only.  The next step then starts with a cold
    cache and pays for no write-back of the flush itself."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.r = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.zero_()
        self.r.sum()
# GroupNorm statistics of the displaced steps (--gn-stats): the method's
# corrected statistics (default) or one of its ablation alternatives
GN_STATS_NAMES = ["corrected", "local", "stale", "sync"]
GN_STATS = 0
# --gn-fuse: GroupNorm -> conv pairs through the conv that normalises its own input
GN_FUSE = False
# the SDXL-shaped workloads' text context is the same at every step (one prompt), so each
# layer's context keys and values are computed at the first step and kept
CTX_FIXED = True


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"),
                "sm_max_mhz": d.get("sm_max_mhz"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# fp32 fused multiply-adds per clock per SM (4 sub-partitions x 32 lanes) and the SM
# count of a B200: the peak of a kernel bound by fp32 CUDA-core arithmetic is
# 148 * 128 * 2 flops * the SM clock (74.4 TFLOP/s at 1965 MHz)
FP32_FMA_PER_CLK_PER_SM, B200_SMS = 128, 148


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
            "unet_mini": B.UNET_MINI, "transformer": B.TRANSFORMER, "unet_sdxl": B.UNET_SDXL}[wl.kind]


def wl_context(wl):
    """(ctx_len, ctx_dim, ff_inner) of a transformer or whole-U-Net workload, else None."""
    if wl.kind == "transformer":
        return (wl.ctx_len, wl.ctx_dim, wl.ff_inner)
    return (wl.ctx_len, wl.ctx_dim, 0) if wl.kind == "unet_sdxl" else None


def oracle_context(wl):
    """A transformer workload's text context for the oracle (fp64), else None."""
    from displaced_patch_parallelism_b200 import synth
    return synth.context(wl).double().numpy() if wl.kind == "transformer" else None


def block_desc(B, wl, H=None):
    d = B.dp_block_desc_init(block_kind(B, wl), H or wl.H, wl.W, wl.C, wl.cout, wl.G, wl.P,
                             wl.heads, B.BF16 if wl.dtype == "bf16" else B.FP32, wl.silu,
                             wl.eps, 1.0)
    if wl.kind == "unet_sdxl":
        B.dp_block_desc_set_unet(d, wl.base, *wl.depths)
        B.dp_block_desc_set_time_embedding(d, wl.temb_dim)
    if wl.kind == "transformer":
        B.dp_block_desc_set_depth(d, wl.depth)
    if wl_context(wl):
        B.dp_block_desc_set_context(d, *wl_context(wl))
        if CTX_FIXED:
            B.dp_block_desc_set_context_fixed(d, True)
    B.dp_block_desc_set_gn_stats(d, GN_STATS)
    if GN_FUSE:
        B.dp_block_desc_set_gn_fusion(d, 1)
    return d


def launch_plan(B, wl, mode):
    """(kernel, algorithmic flops, algorithmic bytes) of every launch of one block step,
    as the library reports them from the step's own code path."""
    d = block_desc(B, wl)
    return [B.dp_block_launch_info(d, mode, i) for i in range(B.dp_block_launch_count(d))]


L2_BYTES = 126 << 20          # B200 L2


def wl_flops(wl, H=None):
    """Algorithmic flops of one displaced step of workload ``wl`` (rows ``H`` if given): the
    convolutions, projections and attention contractions, multiply-adds counted twice.
    Computed from the shapes alone, so the oracle arm never loads the CUDA library."""
    H = H or wl.H
    hw = float(H) * wl.W
    C, Co = float(wl.C), float(wl.cout)

    def conv(hw_out, ci, co):
        return 2.0 * hw_out * co * 9.0 * ci

    def resblock(hw_, ci, co):
        return conv(hw_, ci, co) + conv(hw_, co, co) + (2.0 * hw_ * co * ci if ci != co else 0.0)

    def attn(t, c):
        return 2.0 * t * 3.0 * c * c + 4.0 * t * t * c + 2.0 * t * c * c

    if wl.kind == "gn_conv":
        return conv(hw, C, Co)
    if wl.kind == "resblock":
        return resblock(hw, C, Co)
    if wl.kind == "attn":
        return attn(hw, C)
    def transformer(t, c, f, depth):
        Tk, Cc = float(wl.ctx_len), float(wl.ctx_dim)
        ctx_kv = 0.0 if CTX_FIXED else 2.0 * Tk * 2.0 * c * Cc   # kept from the first step
        layer = (2.0 * t * c * c * 3.0 + 2.0 * t * 3.0 * c * c + 4.0 * t * t * c + ctx_kv +
                 4.0 * t * Tk * c + 2.0 * t * 2.0 * f * c + 2.0 * t * c * f)
        return 2.0 * t * c * c * 2.0 + depth * layer

    if wl.kind == "transformer":
        return transformer(hw, C, float(wl.ff_inner), wl.depth)
    if wl.kind == "unet_sdxl":
        from displaced_patch_parallelism_b200 import synth
        level = {"d0": 0, "u0": 0, "d1": 1, "u1": 1, "d2": 2, "u2": 2, "mid": 2}
        depth = {"d0": wl.depths[0], "u0": wl.depths[0], "d1": wl.depths[1], "u1": wl.depths[1],
                 "d2": wl.depths[2], "u2": wl.depths[2], "mid": wl.depths[2]}
        total = 0.0
        for kind, pre, ci, co in synth.sdxl_unet_stages(wl.base, wl.depths):
            key = pre.split(".")[0]
            t = hw / 4 ** level.get(key, 0)          # the stage's pixels (its input's, for down/up)
            if kind == "conv_in":
                total += conv(hw, C, co)
            elif kind == "out":
                total += conv(hw, ci, C)
            elif kind == "down":
                total += conv(t / 4, ci, co)
            elif kind == "up":
                total += conv(t * 4, ci, co)
            elif kind == "resblock":
                total += resblock(t, ci, co) + 2.0 * co * wl.temb_dim
            else:
                total += transformer(t, ci, 4.0 * ci, depth[key])
        return total
    if wl.kind == "unet_mini":
        return (conv(hw, C, 320) + resblock(hw, 320, 320) + conv(hw / 4, 320, 320) +
                resblock(hw / 4, 320, 640) + attn(hw / 4, 640) + conv(hw / 16, 640, 640) +
                resblock(hw / 16, 640, 1280) + attn(hw / 16, 1280))
    raise ValueError(wl.kind)


def crop_rows_for(wl, seconds_per_step):
    """Rows per band of a row crop whose displaced oracle step takes about
    ``seconds_per_step`` on this host (attention blocks keep the whole image: their
    tiles need every token)."""
    import dataclasses
    hb = wl.H // wl.P
    if wl.kind in ("attn", "transformer"):
        return wl, hb
    t_small = oracle_step_time(dataclasses.replace(wl, H=wl.P * 2))[0]
    per_row = t_small / (2 * wl.P)
    rows = max(2, min(hb, int(seconds_per_step / max(per_row, 1e-6) / wl.P)))
    return dataclasses.replace(wl, H=wl.P * rows), rows


def oracle_step_time(w):
    """One sync step, then one timed displaced step of the oracle on workload ``w``."""
    from displaced_patch_parallelism_b200 import synth
    from oracle import dp_oracle as O
    ctx = oracle_context(w)
    wts = {n: v.double().numpy() for n, v in synth.make_weights(w).items()}
    xs = synth.InputStream(w)
    st = {}
    O.block_step(w.kind, st, xs.x(0)[0], wts, w.P, w.G, w.eps, 1.0, synth.SYNC, w.dtype,
                 heads=w.heads, silu=w.silu, ctx=ctx)
    t0 = time.perf_counter()
    O.block_step(w.kind, st, xs.x(1)[0], wts, w.P, w.G, w.eps, 1.0, synth.DISPLACED, w.dtype,
                 heads=w.heads, silu=w.silu, gn_stats=GN_STATS, ctx=ctx)
    return time.perf_counter() - t0, wts, st, xs, ctx


def cpu_baseline_ours(wl, seconds):
    """The oracle, as it stands, on this host: displaced steps of a row crop of the workload
    (each about a quarter of ``seconds``) until ``seconds`` pass.  Returns the line's
    ``cpu_baseline`` object."""
    from displaced_patch_parallelism_b200 import synth
    from oracle import dp_oracle as O
    w, rows = crop_rows_for(wl, seconds / 4)
    _, wts, st, xs, ctx = oracle_step_time(w)
    x = xs.x(2)[0]
    reps, t0 = 0, time.perf_counter()
    while True:
        O.block_step(w.kind, st, x, wts, w.P, w.G, w.eps, 1.0, synth.DISPLACED, w.dtype,
                     heads=w.heads, silu=w.silu, gn_stats=GN_STATS, ctx=ctx)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    fl = wl_flops(wl, w.H)
    return {"value": round(fl * reps / el / 1e12, 6), "unit": "TFLOP/s",
            "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
            "sample": (f"{reps} displaced steps of {wl.name} on a {w.C}x{w.H}x{w.W} row crop "
                       f"({rows} rows per band, {fl / 1e9:.2f} GFLOP each) in {el:.1f} s")}


def run_reference(args, wl):
    """The CPU oracle on the host cores: each step a displaced step of a row crop of the block."""
    from displaced_patch_parallelism_b200 import synth
    from oracle import dp_oracle as O
    budget = 150.0
    cores = len(os.sched_getaffinity(0))
    w, rows = crop_rows_for(wl, budget / max(1, args.steps + args.warmup))
    _, wts, st, xs, ctx = oracle_step_time(w)
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
            "config": workload_config(wl, ws=1, extra={"sample": sample}),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def input_bytes(wl):
    return wl.C * wl.H * wl.W * (2 if wl.dtype == "bf16" else 4)


def l2_policy(wl):
    """(flush between steps?, description): a step whose input alone exceeds L2 evicts it
    by itself; smaller ones get a 256 MiB write between steps, outside the timed events."""
    if input_bytes(wl) > L2_BYTES:
        return False, (f"inputs larger than L2 ({input_bytes(wl) / 1e6:.1f} MB input per step, "
                       f"4 inputs in rotation); no flush")
    return True, ("flushed between steps (256 MiB write, then a 256 MiB read that writes the dirty "
                  "lines back; both outside the timed events)")


def workload_config(wl, ws, extra=None):
    cfg = {"workload": wl.name, "shape_nchw": [1, wl.C, wl.H, wl.W], "P": wl.P,
           "mode": "displaced", "gn_stats": GN_STATS_NAMES[GN_STATS],
           "gn_conv": "fused (conv normalises its input)" if GN_FUSE else "separate passes",
           "l2": l2_policy(wl)[1],
           "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU"}
    if wl.dtype == "fp32":
        cfg["arithmetic"] = "fp32 storage and arithmetic; the conv on the CUDA cores"
    if wl.kind in ("transformer", "unet_sdxl"):
        cfg["context"] = ("fixed: each layer's context keys and values computed at the first step "
                          "and kept" if CTX_FIXED else "context keys and values recomputed every step")
    cfg.update(extra or {})
    return cfg


class Run:
    """One workload's block, weights and inputs on the device."""

    def __init__(self, wl, dev, pool=4):
        import torch

        from displaced_patch_parallelism_b200 import binding as B
        from displaced_patch_parallelism_b200 import synth
        from displaced_patch_parallelism_b200.weights import block_weights, unet_sdxl_weights
        self.wl, self.B = wl, B
        self.tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
        if wl.kind == "unet_sdxl":
            # 2.56 billion parameters: drawn on the device; the step's context and time
            # embedding are its last two pointers
            wts = synth.make_weights(wl, device=dev)
            self.dw = unet_sdxl_weights(wts, synth.sdxl_unet_stages(wl.base, wl.depths), wl.depths,
                                        self.tdt, dev)
            del wts
            self.dw += [synth.context(wl).to(self.tdt).to(dev),
                        synth.randn((wl.temb_dim,), wl.seed + 600).to(dev)]
        else:
            wts = synth.make_weights(wl)
            self.dw = block_weights(wl.kind, wts, self.tdt, dev, depth=wl.depth)
            if wl.kind == "transformer":     # the step's text context is the last pointer
                self.dw.append(synth.context(wl).to(self.tdt).to(dev))
        unet = (wl.base,) + tuple(wl.depths) if wl.kind == "unet_sdxl" else None
        self.blk = B.Block(block_kind(B, wl), wl.H, wl.W, wl.C, wl.cout, wl.G, wl.P, wl.heads,
                           B.BF16 if wl.dtype == "bf16" else B.FP32, wl.silu, wl.eps, 1.0,
                           device=dev, gn_stats=GN_STATS, context=wl_context(wl), gn_fuse=GN_FUSE,
                           temb_dim=wl.temb_dim if wl.kind == "unet_sdxl" else 0, unet=unet,
                           depth=wl.depth if wl.kind == "transformer" else 1,
                           context_fixed=CTX_FIXED and wl_context(wl) is not None)
        xs = synth.InputStream(wl)
        self.pool = pool
        self.host_x = [synth.nchw_to_nhwc(xs.x(k)).to(self.tdt).pin_memory() for k in range(pool)]
        self.dev_x = [h.to(dev) for h in self.host_x]
        Ho, Wo = (wl.H // 4, wl.W // 4) if wl.kind == "unet_mini" else (wl.H, wl.W)
        self.out = torch.empty(Ho, Wo, wl.cout, dtype=self.tdt, device=dev)
        self.flush_between = l2_policy(wl)[0]
        self.plan = launch_plan(B, wl, B.DISPLACED)
        assert len(self.plan) == self.blk.launches
        self.flops = wl_flops(wl)

    def warm(self, n):
        import torch
        for i in range(n):
            self.blk.step(self.dev_x[i % self.pool], self.out, self.dw,
                          self.B.dp_mode_for_step(i, self.wl.warmup))
        torch.cuda.synchronize()


def time_steps(run, steps, flush, dist, sampler=None):
    """Device time (ms) of each of ``steps`` displaced steps, an event pair around each."""
    import torch
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for e in ev0 + ev1:          # torch creates the CUDA event on its first record
        e.record()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    wall0 = time.perf_counter()
    for k in range(steps):
        if run.flush_between:
            flush()
        ev0[k].record()
        run.blk.step(run.dev_x[k % run.pool], run.out, run.dw, run.B.DISPLACED)
        ev1[k].record()
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    clocks = sampler.stop() if sampler else None
    if dist:
        dist.barrier()
    return [ev0[k].elapsed_time(ev1[k]) for k in range(steps)], wall, clocks


def time_graph(run, steps, flush):
    """Device time (ms) of ``steps`` displaced steps replayed from the library's CUDA graphs
    (dp_block_graph_*: one captured step per ping-pong parity, the first input buffer fixed in
    them), an event pair around each, L2 flushed between steps as in time_steps."""
    import torch
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    with torch.cuda.stream(s):
        g = run.blk.graph(run.dev_x[0], run.out, run.dw, run.B.DISPLACED, s)
        g.launch(s)                      # first replay: uploads the graphs
        for k in range(steps):
            if run.flush_between:
                flush()
            ev[k][0].record(s)
            g.launch(s)
            ev[k][1].record(s)
    torch.cuda.synchronize()
    g.close()
    return [a.elapsed_time(b) for a, b in ev]


def breakdown(run, steps, flush, peaks):
    """Per-kernel roles of the step: mean duration, share, rate; and the dominant role's
    roofline.  An event before every launch (dp_block_step_timed) keeps kernels from
    overlapping, so these times add up to a little more than the step."""
    import torch
    n_launch = run.blk.launches
    n_bd = min(steps, 50)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(n_launch + 1)]
              for _ in range(n_bd)]
    for row in events:
        for e in row:
            e.record()
    torch.cuda.synchronize()
    for k in range(n_bd):
        if run.flush_between:
            flush()
        run.blk.step_timed(run.dev_x[k % run.pool], run.out, run.dw, run.B.DISPLACED, events[k])
    torch.cuda.synchronize()
    per_launch = [[events[k][i].elapsed_time(events[k][i + 1]) for i in range(n_launch)]
                  for k in range(n_bd)]
    roles = [r for r, _, _ in run.plan]
    work = [(f, b) for _, f, b in run.plan]
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
    src = {"conv": ["dp_gemm.cu"], "conv_gn": ["dp_gemm.cu"], "linear": ["dp_gemm.cu"],
           "attn": ["dp_attn.cu"],
           "gn_stats": ["dp_gn.cu"], "gn_apply": ["dp_gn.cu"], "gn_fused": ["dp_gn.cu"],
           "gn_cluster": ["dp_gn.cu"], "copy": ["dp_refresh.cu"],
           "conv_small": ["dp_conv_small.cu"], "splitk_finish": ["dp_gemm.cu"],
           "conv_f32": ["dp_conv_f32.cu"],
           "layernorm": ["dp_token.cu"], "geglu": ["dp_token.cu"], "temb": ["dp_temb.cu"],
           "conv_narrow": ["dp_conv_narrow.cu"], "concat": ["dp_resample.cu"],
           "upsample": ["dp_resample.cu"]}
    traffic = load_traffic(f"{dominant}:{run.wl.name}", kernel_source_hash(src[dominant]))
    if dk["tflops"] and dominant in ("conv_f32", "conv_small"):
        sm_mhz = peaks.get("sm_max_mhz") or 1965.0
        alu_peak = B200_SMS * FP32_FMA_PER_CLK_PER_SM * 2 * sm_mhz * 1e6 / 1e12
        roof = {"bound": "alu", "achieved": dk["tflops"], "peak": round(alu_peak, 1), "unit": "TFLOP/s",
                "frac": round(dk["tflops"] / alu_peak, 4), "traffic": traffic, "kernel": dominant,
                "peak_source": "derived: 148 SMs x 128 fp32 FMA/clk x 2 flops x max SM clock"}
    elif dk["tflops"]:
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
    return kernels, roof, gn


def time_e2e(run, steps, dist, dev):
    """End to end through the public call: every step copies its input from pinned host
    memory, runs the block step and copies its result back to pinned host memory.  The
    copies run on their own streams (the copy engines), so step k+1's input and step k's
    result move while a neighbouring step computes.  Timed on the device from the first
    copy to the last; nothing else (no L2 flush) runs in the timed region."""
    import torch
    s_comp, s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    xin = [torch.empty_like(run.dev_x[0]) for _ in range(2)]
    outb = [torch.empty_like(run.out) for _ in range(2)]
    host_o = [torch.empty(run.out.shape, dtype=run.tdt).pin_memory() for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(steps)]
    ev_comp = [torch.cuda.Event() for _ in range(steps)]
    ev_out = [torch.cuda.Event() for _ in range(steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    t_start.record(s_comp)
    s_in.wait_event(t_start)
    for k in range(steps):
        b = k & 1
        if k >= 2:
            s_in.wait_event(ev_comp[k - 2])      # step k-2 has read xin[b]
        with torch.cuda.stream(s_in):
            xin[b].copy_(run.host_x[k % run.pool], non_blocking=True)
            ev_in[k].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev_in[k])
            if k >= 2:
                s_comp.wait_event(ev_out[k - 2])  # outb[b] has reached the host
            run.blk.step(xin[b], outb[b], run.dw, run.B.DISPLACED)
            ev_comp[k].record(s_comp)
        s_out.wait_event(ev_comp[k])
        with torch.cuda.stream(s_out):
            host_o[b].copy_(outb[b], non_blocking=True)
            ev_out[k].record(s_out)
    s_comp.wait_event(ev_out[steps - 1])
    t_end.record(s_comp)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(t_start.elapsed_time(t_end), dist, dev)
    if dist:
        dist.barrier()
    return e2e_ms, (run.dev_x[0].numel() * run.dev_x[0].element_size(),
                    run.out.numel() * run.out.element_size())


EXTRA_WORKLOADS = ["tiny_fp32_gn_conv", "resblock_320x128x128", "attn_640x64x64",
                   "unet_mini_4x128x128", "transformer_640x64x64", "transformer_1280x32x32",
                   "unet_sdxl_4x128x128"]


def run_ours(args, wl):
    import torch

    from displaced_patch_parallelism_b200 import binding as B
    from displaced_patch_parallelism_b200 import synth

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dist = None
    if ws > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    flush = L2Flush(dev)
    peaks = load_peaks()

    run = Run(wl, dev)
    run.warm(max(args.warmup, wl.warmup + 1))
    step_ms, wall, clocks = time_steps(run, args.steps, flush, dist, ClockSampler(local))
    total_ms = max_over_ranks(sum(step_ms), dist, dev)
    kernels, roof, gn = breakdown(run, args.steps, flush, peaks)
    e2e_ms, (h2d, d2h) = time_e2e(run, args.steps, dist, dev)
    status = B.dp_device_status()
    n_launch = run.blk.launches
    line = {"metric": METRIC, "value": round(job_tflops(ws, run.flops, args.steps, total_ms), 3),
            "unit": "TFLOP/s", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total_ms / args.steps, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
            "config": workload_config(wl, ws),
            "roofline": roof, "kernels": kernels, "groupnorm": gn,
            "e2e": {"value": round(job_tflops(ws, run.flops, args.steps, e2e_ms), 3),
                    "unit": "TFLOP/s", "ms_per_step": round(e2e_ms / args.steps, 5),
                    "copies": "input and result copies on their own streams, overlapping "
                              "neighbouring steps; no L2 flush in the timed region",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": n_launch * args.steps, "clocks": clocks,
            "wall_s_timed_region": round(wall, 4), "device_status": status}
    del run
    torch.cuda.empty_cache()

    # the other workloads: device-timed steps and the per-kernel breakdown
    if not args.headline_only:
        extra = {}
        for name in EXTRA_WORKLOADS:
            if name == wl.name:
                continue
            w = synth.WORKLOADS[name]
            try:
                r = Run(w, dev)
                r.warm(max(args.warmup, w.warmup + 1))
                ms, _, _ = time_steps(r, args.steps, flush, dist)
                t_ms = max_over_ranks(sum(ms), dist, dev)
                k, rf, g = breakdown(r, args.steps, flush, peaks)
                g_ms = max_over_ranks(sum(time_graph(r, args.steps, flush)), dist, dev)
            except B.DPError as e:          # a host-side rejection; recorded, not fatal
                extra[name] = {"error": str(e)}
                continue
            extra[name] = {"ms_per_step": round(t_ms / args.steps, 5),
                           "value": round(job_tflops(ws, r.flops, args.steps, t_ms), 3),
                           "unit": "TFLOP/s", "gflop_per_step": round(r.flops / 1e9, 3),
                           "dtype": w.dtype, "config": workload_config(w, ws),
                           "roofline": {kk: rf[kk] for kk in ("bound", "kernel", "achieved",
                                                              "peak", "unit", "frac")},
                           "kernels": k, "groupnorm": g,
                           "graph": {"ms_per_step": round(g_ms / args.steps, 5),
                                     "value": round(job_tflops(ws, r.flops, args.steps, g_ms), 3),
                                     "unit": "TFLOP/s",
                                     "how": "the same steps replayed from dp_block_graph_* CUDA graphs"},
                           "gpu_launches": r.blk.launches * args.steps}
            del r
            torch.cuda.empty_cache()
        line["workloads"] = extra
        line["device_status"] = line["device_status"] or B.dp_device_status()
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_ours(wl, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="gn_conv_320x480x480")
    ap.add_argument("--headline-only", action="store_true",
                    help="time only --workload (skip the other workloads' lines)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--gn-stats", choices=GN_STATS_NAMES, default="corrected",
                    help="GroupNorm statistics of the displaced steps")
    ap.add_argument("--gn-fuse", action="store_true",
                    help="GroupNorm -> conv pairs through the conv that normalises its own input")
    args = ap.parse_args()
    global GN_STATS, GN_FUSE
    GN_STATS = GN_STATS_NAMES.index(args.gn_stats)
    GN_FUSE = args.gn_fuse
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
