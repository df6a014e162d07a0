#!/usr/bin/env python
"""Benchmark of the VDN hybrid attention layer forward (video-to-video).

One step = one pass of the whole hot path (frame stats, per-frame solve and
bidirectional scan, block-sparse softmax with the readout and gate fused,
gated merge) over one batch of the 768p-shaped synthetic workload (B=1,
H=24, d=dv=128, T=60 latent frames, N=4032 tokens per frame, d_out=3072).
Inputs (4.5 GB of q, k, v) are larger than L2, so no flush is needed between
steps.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]

For N > 1 (launched by torchrun) the layer is split over the ranks by heads
(Ulysses sequence parallelism, the pages' multi-GPU setting; strong scaling):
each rank holds a token shard of q, k, v, two NCCL all-to-all exchanges move
q, k, v to head shards and the gated Z back to token shards, and `value`
counts the layer's tokens over the slowest rank's time. `--dp` instead runs
N independent replicas of the layer (weak scaling, no exchange). Timing is
the max over ranks.
"""
import argparse
import json
import math
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "VDN hybrid-layer fwd ms/layer & tokens/s on 1 B200; % of BF16 peak / HBM BW"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DEFAULT_WORKLOAD = "768p"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of SM clock, power and throttle reasons (every 200 ms)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.fh = None

    def start(self):
        self.fh = tempfile.TemporaryFile(mode="w+")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_id), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.seek(0)
        rows = [ln.strip().split(", ") for ln in self.fh if ln.strip()]
        self.fh.close()
        samples = []
        for r in rows:
            try:
                samples.append(dict(sm=float(r[1]), smax=float(r[2]), power=float(r[3]),
                                    hw=r[5].strip(), hw_th=r[6].strip(), sw_th=r[7].strip(),
                                    sw_pc=r[8].strip()))
            except (ValueError, IndexError):
                continue
        if not samples:
            return None
        load = [s for s in samples if s["power"] > 250.0] or samples
        reasons = set()
        for s in load:
            for key, name in (("hw", "hw_slowdown"), ("hw_th", "hw_thermal_slowdown"),
                              ("sw_th", "sw_thermal_slowdown"), ("sw_pc", "sw_power_cap")):
                if s[key] == "Active":
                    reasons.add(name)
        return {"sm_mhz": float(np.median([s["sm"] for s in load])),
                "sm_max_mhz": float(max(s["smax"] for s in samples)),
                "reasons": sorted(reasons), "samples": len(load)}


def _physical_gpu(local_rank):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


# --------------------------------------------------------------- workload
def workload_cfg(name, n_ctx=0):
    from synthetic import get_workload
    import softmax_attention_video_vdn_b200 as vdn
    wl = get_workload(name, n_ctx=n_ctx) if n_ctx else get_workload(name)
    cfg = vdn.make_config(B=wl.B, H=wl.H, T=wl.T, N=wl.N, d=wl.d, dv=wl.dv, dtype=wl.dtype,
                          lam=wl.lam, beta=wl.beta, block_frames=wl.block_frames,
                          window_blocks=wl.window_blocks, anchors=wl.anchors, d_out=wl.d_out,
                          w_per_head=wl.w_per_head, n_ctx=wl.n_ctx)
    return wl, cfg


def workload_name(wl, cfg):
    """The workload string of the JSON line (the same for both arms)."""
    return (f"{wl.name}: B={cfg.B} H={cfg.H} d={cfg.d} dv={cfg.dv} T={cfg.T} N={cfg.N} "
            f"d_out={cfg.d_out}" + (f" n_ctx={cfg.n_ctx}" if cfg.n_ctx else ""))


def softmax_work(cfg):
    """Algorithmic FLOPs of the softmax kernel: QK^T and PV over every allowed
    (query, key) pair (video pairs of the frame mask, every video query with
    every context key, every context query with every key); also the number
    of pairs (= exponentials) and the frame-mask density."""
    import softmax_attention_video_vdn_b200 as vdn
    mask, _ = vdn.vdn_window_plan(cfg)
    TN = cfg.T * cfg.N
    pairs = float(mask.sum()) * cfg.N * cfg.N + 2.0 * TN * cfg.n_ctx + float(cfg.n_ctx) ** 2
    BH = cfg.B * cfg.H
    qk_pv = 2.0 * pairs * (cfg.d + cfg.dv) * BH
    return qk_pv, pairs * BH, float(mask.mean())


def readout_bytes(cfg):
    """Algorithmic HBM bytes of one readout launch: q read, the output rows
    written, the two states per (b, h, block) read."""
    BH = cfg.B * cfg.H
    io = 2 if cfg.dtype == 1 else 4
    return BH * cfg.L * (cfg.d + cfg.dv) * io + 2 * BH * cfg.nb * cfg.dv * cfg.d * 4


def softmax_launches(cfg):
    """Kernel launches of one softmax call: the segments of the frame plan in
    chunks of at most 40 (the plan's per-launch capacity)."""
    import softmax_attention_video_vdn_b200 as vdn
    _, plan = vdn.vdn_window_plan(cfg)
    n_seg, i = 0, 0
    while i < len(plan):
        nr = int(plan[i + 2])
        i += 3 + 2 * nr
        n_seg += 1
    n_seg += 1 if cfg.n_ctx else 0     # the context queries' segment
    return (n_seg + 39) // 40


def measured_traffic(kernel_record):
    """DRAM bytes per launch from a committed ncu record, if the kernel's
    sources are unchanged since the capture; otherwise None."""
    import hashlib
    path = os.path.join(ROOT, "profiles", kernel_record)
    try:
        with open(path) as fh:
            rec = json.load(fh)
        h = hashlib.sha256()
        for src in rec["sources"]:
            with open(os.path.join(ROOT, src), "rb") as fh:
                h.update(fh.read())
    except (OSError, ValueError, KeyError):
        return None
    if h.hexdigest() != rec.get("source_sha256"):
        return None
    return float(rec["traffic_bytes_per_launch"])


def stats_bytes(cfg):
    """Algorithmic HBM bytes of one frame-stats launch: k, v read once, G, C written."""
    BH = cfg.B * cfg.H
    return BH * cfg.L * (cfg.d + cfg.dv) * 2 + BH * cfg.T * (cfg.d * cfg.d + cfg.dv * cfg.d) * 4


# ------------------------------------------------------------ multi-rank
def rank_workload(wl, rank):
    """Each rank runs its own batch of the same shape (weak scaling): same
    workload, seed offset by the rank so the ranks' inputs differ."""
    return wl.with_(seed=wl.seed + 1000 * rank)


def max_over_ranks(values, world, device="cpu"):
    """Element-wise maximum of per-rank timings (ms) across the process group."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


# -------------------------------------------------------------------- ours
def run_ours(args, rank, world, local_rank):
    import torch.distributed as dist

    import softmax_attention_video_vdn_b200 as vdn
    from softmax_attention_video_vdn_b200 import build as vbuild
    from softmax_attention_video_vdn_b200.layer import HybridLayer, io_dtype
    from synthetic import make_inputs

    vbuild.build()
    vdn.load_library()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl, cfg = workload_cfg(args.workload, args.n_ctx)
    wl = rank_workload(wl, rank)
    x = make_inputs(wl, device=dev)
    q, k, v, gate = (x[n] for n in ("q", "k", "v", "gate_logits"))
    W1, W2 = x.get("W1"), x.get("W2")
    fp8 = bool(getattr(args, "fp8", False)) and wl.softmax
    layer = HybridLayer(cfg, dev, fp8=fp8) if wl.softmax else None
    stream = torch.cuda.current_stream(dev)
    status = layer.status if layer else torch.zeros(1, dtype=torch.int32, device=dev)

    if wl.softmax:
        G, C, S_fwd, S_bwd, Z, scan_ws, sm_ws = _layer_views(cfg, layer, dev)
        # the same kernels as vdn_hybrid_forward(_fp8), one entry point per
        # stage so that each kernel is timed on its own
        if fp8:
            u8 = dict(dtype=torch.uint8, device=dev)
            x8 = [torch.empty(t.shape, **u8) for t in (q, k, v)]
            sc = torch.empty((3, cfg.B * cfg.H), dtype=torch.float32, device=dev)
            qws = torch.empty(vdn.vdn_workspace_size(cfg, vdn.VDN_WS_QUANT), **u8)

            def quantize():
                for i, t in enumerate((q, k, v)):
                    vdn.vdn_quantize_fp8(cfg, t, x8[i], sc[i], qws, stream)
            stages = ["frame_stats", "solve_scan", "quantize", "softmax_window", "readout",
                      "gated_merge"]
            calls = [
                lambda: vdn.vda_frame_stats(cfg, k, v, G, C, stream),
                lambda: vdn.vda_bidir_scan(cfg, G, C, S_fwd, S_bwd, scan_ws, status, stream),
                quantize,
                lambda: vdn.vdn_softmax_window_fp8(cfg, x8[0], x8[1], x8[2], sc[0], sc[1], sc[2],
                                                   gate, Z, sm_ws, status, stream),
                lambda: vdn.vda_readout_gated(cfg, q, S_fwd, S_bwd, gate, Z, stream),
                lambda: vdn.vdn_gated_merge(cfg, Z, W1, W2, layer.Y, stream),
            ]
        else:
            stages = ["frame_stats", "solve_scan", "softmax_window", "readout", "gated_merge"]
            calls = [
                lambda: vdn.vda_frame_stats(cfg, k, v, G, C, stream),
                lambda: vdn.vda_bidir_scan(cfg, G, C, S_fwd, S_bwd, scan_ws, status, stream),
                lambda: vdn.vdn_softmax_window(cfg, q, k, v, None, None, gate, Z, sm_ws, status,
                                               stream),
                lambda: vdn.vda_readout_gated(cfg, q, S_fwd, S_bwd, gate, Z, stream),
                lambda: vdn.vdn_gated_merge(cfg, Z, W1, W2, layer.Y, stream),
            ]
    else:  # linear branch only: statistics, scan, readout
        f32 = dict(dtype=torch.float32, device=dev)
        G = torch.empty((cfg.B, cfg.H, cfg.T, cfg.d, cfg.d), **f32)
        C = torch.empty((cfg.B, cfg.H, cfg.T, cfg.dv, cfg.d), **f32)
        S_fwd = torch.empty((cfg.B, cfg.H, cfg.nb, cfg.dv, cfg.d), **f32)
        S_bwd = torch.empty_like(S_fwd)
        scan_ws = torch.empty(vdn.vdn_workspace_size(cfg, vdn.VDN_WS_SCAN), dtype=torch.uint8,
                              device=dev)
        o_lin = torch.empty((cfg.B, cfg.L, cfg.H, cfg.dv), dtype=io_dtype(cfg), device=dev)
        stages = ["frame_stats", "solve_scan", "readout"]
        calls = [
            lambda: vdn.vda_frame_stats(cfg, k, v, G, C, stream),
            lambda: vdn.vda_bidir_scan(cfg, G, C, S_fwd, S_bwd, scan_ws, status, stream),
            lambda: vdn.vda_readout(cfg, q, S_fwd, S_bwd, o_lin, stream),
        ]

    def step(ev=None):
        for i, call in enumerate(calls):
            if ev:
                ev[i].record(stream)
            call()
        if ev:
            ev[len(calls)].record(stream)

    def check(where):
        st = vdn.vdn_read_status(status, stream)
        if st != 0:
            raise RuntimeError(f"device status {where}: {vdn.vdn_status_string(st)}")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    check("after warm-up")

    n_ev = len(calls) + 1
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    clocks = ClockSampler(_physical_gpu(local_rank))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    time.sleep(0.3)
    for i in range(args.steps):
        step(evs[i])
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    per = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(len(calls))]
                    for i in range(args.steps)])  # ms
    step_ms = float(per.sum(axis=1).mean())
    check("after timing")

    e2e = None
    if wl.softmax and not args.no_e2e:
        fwd = vdn.vdn_hybrid_forward_fp8 if layer.fp8 else vdn.vdn_hybrid_forward

        def run_layer(ins, Y):
            fwd(cfg, ins[0], ins[1], ins[2], gate, W1, W2, Y, layer.ws, layer.status, stream)

        e2e = _e2e(args, (q, k, v), layer.Y, run_layer, stream, dev, world)
        st = layer.check_status(stream)
        if st != 0:
            raise RuntimeError(f"device status after end-to-end run: {vdn.vdn_status_string(st)}")
    e2e_ms = e2e["ms"] if e2e else 0.0
    step_ms, e2e_ms = max_over_ranks([step_ms, e2e_ms], world, dev)
    tokens = cfg.B * cfg.L * world
    if rank != 0:
        return None
    peaks, peak_src = load_peaks()
    ms = {n: float(per[:, i].mean()) for i, n in enumerate(stages)}
    kern = {n: {"ms": ms[n]} for n in stages}
    kern["frame_stats"]["GB/s"] = stats_bytes(cfg) / (ms["frame_stats"] * 1e-3) / 1e9
    kern["readout"]["GB/s"] = readout_bytes(cfg) / (ms["readout"] * 1e-3) / 1e9
    roof = None
    if wl.softmax:
        flops, _, density = softmax_work(cfg)
        achieved = flops / (ms["softmax_window"] * 1e-3) / 1e12
        kern["softmax_window"]["TFLOP/s"] = achieved
        # per token: 2*H*dv inputs times d_out outputs (shared weights: per head)
        mflops = 2.0 * cfg.B * cfg.L * 2 * cfg.H * cfg.dv * cfg.d_out
        kern["gated_merge"]["TFLOP/s"] = mflops / (ms["gated_merge"] * 1e-3) / 1e12
        if cfg.dtype == vdn.VDN_BF16 and fp8:
            # e4m3 dense peak = the measured bf16 peak x the nominal ratio 4.5 / 2.25
            peak = 2.0 * float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
            roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": None,
                    "kernel": "softmax_window_fp8_kernel",
                    "peak_source": f"{peak_src} bf16_tflops_sustained x 2 (e4m3 / bf16 nominal)"}
            qbytes = 3 * cfg.B * cfg.H * cfg.L * cfg.d * (2 + 2 + 1)
            kern["quantize"]["GB/s"] = qbytes / (ms["quantize"] * 1e-3) / 1e9
        elif cfg.dtype == vdn.VDN_BF16:
            peak = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
            roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak,
                    "traffic": (measured_traffic("softmax_window_768p_traffic.json")
                                if args.workload == "768p" else None),
                    "kernel": "softmax_window_bf16_kernel",
                    "peak_source": f"{peak_src} bf16_tflops_sustained"}
    else:
        density = None
        hbm = float(peaks["hbm_gbs"])
        gbs = kern["frame_stats"]["GB/s"]
        roof = {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                "traffic": None, "kernel": "frame_stats_bf16_kernel",
                "peak_source": f"{peak_src} hbm_gbs"}
    result = {
        "metric": METRIC, "value": tokens / (step_ms * 1e-3), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": "e4m3 softmax, bf16 elsewhere" if fp8 else {0: "f32", 1: "bf16"}[cfg.dtype],
        "data": "synthetic",
        "config": {"workload": workload_name(wl, cfg),
                   "tokens_per_layer": cfg.B * cfg.L, "mask_density": density,
                   "l2": "inputs larger than L2" if 3 * q.numel() * q.element_size() > 126e6
                         else "inputs smaller than L2",
                   "parallelism": f"dp{world}" if world > 1 else "single"},
        "e2e": ({"value": tokens / (e2e_ms * 1e-3), "unit": UNIT,
                 "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                 "how": "vdn_hybrid_forward from pinned host q,k,v; copies on two "
                        "streams, double-buffered, overlapping the previous/next step"}
                if e2e else None),
        # stats 1, solve + scan 2, softmax (per plan chunk), readout 1, merge 1,
        # and with e4m3 two quantiser launches per tensor
        "gpu_launches": ((5 + softmax_launches(cfg) + (6 if fp8 else 0)) if wl.softmax else 4)
                        * args.steps,
        "roofline": roof,
        "kernels": kern,
        "clocks": clk,
    }
    return result


def run_ulysses(args, rank, world, local_rank):
    """One 768p layer split over the ranks by heads (Ulysses sequence
    parallelism, strong scaling): each rank holds a token shard of q, k, v,
    re-shards them by head (NCCL all-to-all), runs the hybrid path on its
    H/world heads, re-shards Z back by tokens and runs the merge on its token
    rows. One step = one forward of the whole layer; `value` counts the
    layer's tokens over the slowest rank's time."""
    import torch.distributed as dist

    import softmax_attention_video_vdn_b200 as vdn
    from softmax_attention_video_vdn_b200 import build as vbuild
    from softmax_attention_video_vdn_b200.ulysses import STAGES, UlyssesLayer
    from synthetic import make_inputs

    vbuild.build()
    vdn.load_library()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl, cfg = workload_cfg(args.workload, args.n_ctx)
    if not wl.softmax or wl.dtype != "bf16":
        raise SystemExit("the head-sharded layer runs bf16 workloads with a softmax branch")
    layer = UlyssesLayer(cfg, device=dev)
    Ls = layer.Ls
    # every rank draws the same full input (same seed) and keeps its token shard
    x = make_inputs(wl, device=dev)
    shard = [x[n][:, :, rank * Ls:(rank + 1) * Ls].permute(0, 2, 1, 3).contiguous()
             for n in ("q", "k", "v")]
    gate, W1, W2 = x["gate_logits"], x["W1"], x["W2"]
    del x
    torch.cuda.empty_cache()
    stream = torch.cuda.current_stream(dev)

    def step(ev=None, Y=None):
        layer.forward(shard[0], shard[1], shard[2], gate, W1, W2, stream=stream, Y=Y, events=ev)

    def check(where):
        st = vdn.vdn_read_status(layer.status, stream)
        if st != 0:
            raise RuntimeError(f"device status {where}: {vdn.vdn_status_string(st)}")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    check("after warm-up")
    n_ev = len(STAGES) + 1
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    clocks = ClockSampler(_physical_gpu(local_rank))
    dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    time.sleep(0.3)
    for i in range(args.steps):
        step(evs[i])
    torch.cuda.synchronize(dev)
    dist.barrier()
    clk = clocks.stop()
    per = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(len(STAGES))]
                    for i in range(args.steps)])
    step_ms = float(per.sum(axis=1).mean())
    stage_ms = [float(per[:, j].mean()) for j in range(len(STAGES))]
    check("after timing")
    e2e = None
    if not args.no_e2e:
        e2e = _e2e(args, shard, layer.Y,
                   lambda ins, Y: layer.forward(ins[0], ins[1], ins[2], gate, W1, W2,
                                                stream=stream, Y=Y),
                   stream, dev, world)
        check("after the end-to-end steps")
    e2e_ms = e2e["ms"] if e2e else 0.0
    # every rank's stage times; the slowest rank's step
    mx = max_over_ranks([step_ms, e2e_ms] + stage_ms, world, dev)
    step_ms, e2e_ms, stage_ms = mx[0], mx[1], mx[2:]
    if rank != 0:
        return None
    peaks, peak_src = load_peaks()
    ms = dict(zip(STAGES, stage_ms))
    kern = {n: {"ms": ms[n]} for n in STAGES}
    ch = layer.cfg_heads
    flops, _, density = softmax_work(ch)
    achieved = flops / (ms["softmax_window"] * 1e-3) / 1e12
    kern["softmax_window"]["TFLOP/s"] = achieved
    kern["frame_stats"]["GB/s"] = stats_bytes(ch) / (ms["frame_stats"] * 1e-3) / 1e9
    kern["readout"]["GB/s"] = readout_bytes(ch) / (ms["readout"] * 1e-3) / 1e9
    mflops = 2.0 * cfg.B * Ls * 2 * cfg.H * cfg.dv * cfg.d_out
    kern["gated_merge"]["TFLOP/s"] = mflops / (ms["gated_merge"] * 1e-3) / 1e12
    # bytes each rank sends and receives in the two exchanges (its shard of
    # q, k, v less its own heads; its heads' Z less its own tokens)
    xbytes = (3 * cfg.B * Ls * cfg.H * cfg.d * 2 + cfg.B * cfg.L * 2 * layer.Hs * cfg.dv * 2)
    xbytes *= (world - 1) / world
    kern["reshard_qkv"]["note"] = ("k, v layout copy + NCCL all-to-all per (batch, local head); q's "
                                   "layout copy, its exchange overlapping frame_stats and solve_scan")
    kern["reshard_z"]["note"] = "NCCL all-to-all per batch item, no copy"
    peak = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
    roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "traffic": None, "kernel": "softmax_window_bf16_kernel",
            "peak_source": f"{peak_src} bf16_tflops_sustained",
            "work": f"this rank's {layer.Hs} heads"}
    tokens = cfg.B * cfg.L
    return {
        "metric": METRIC, "value": tokens / (step_ms * 1e-3), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": workload_name(wl, cfg), "tokens_per_layer": tokens,
                   "mask_density": density, "l2": "inputs larger than L2",
                   "parallelism": f"ulysses{world}", "heads_per_gpu": layer.Hs,
                   "exchange_bytes_per_rank": xbytes},
        "e2e": ({"value": tokens / (e2e_ms * 1e-3), "unit": UNIT,
                 "h2d_bytes_per_step": e2e["h2d"] * world, "d2h_bytes_per_step": e2e["d2h"] * world,
                 "how": "each rank: its token shard of q, k, v from pinned host memory, "
                        "UlyssesLayer.forward, its rows of Y back; copies double-buffered on "
                        "their own streams"}
                if e2e else None),
        # stats 1, solve + scan 2, softmax (per plan chunk), readout 1, merge 1
        "gpu_launches": (5 + softmax_launches(ch)) * args.steps,
        "roofline": roof,
        "kernels": kern,
        "clocks": clk,
    }


BWD_METRIC = "VDN hybrid-layer bwd ms/layer & tokens/s on 1 B200; % of BF16 peak"


def backward_launches(cfg):
    """Kernel launches of one vdn_hybrid_backward: merge dgrad and wgrad, the
    preparation kernel, the linear branch (stats, solve, scan, readout, stats
    of do, block sums, adjoint scan, per-frame grads, stats backward) and two
    softmax kernels per plan chunk."""
    return 2 + 1 + 9 + 2 * softmax_launches(cfg)


def run_backward(args, rank, world, local_rank):
    """The layer backward (vdn_hybrid_backward) on the forward's saved Z and
    lse, one step = one backward over the whole layer; plus each part timed
    through its own entry point."""
    import torch.distributed as dist

    import softmax_attention_video_vdn_b200 as vdn
    from softmax_attention_video_vdn_b200 import build as vbuild
    from softmax_attention_video_vdn_b200.layer import HybridLayerTrain
    from synthetic import make_inputs

    vbuild.build()
    vdn.load_library()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl, cfg = workload_cfg(args.workload, args.n_ctx)
    wl = rank_workload(wl, rank)
    x = make_inputs(wl, device=dev)
    q, k, v, gate, W1, W2 = (x[n] for n in ("q", "k", "v", "gate_logits", "W1", "W2"))
    stream = torch.cuda.current_stream(dev)
    layer = HybridLayerTrain(cfg, dev)
    layer.forward(q, k, v, gate, W1, W2, stream)
    gen = torch.Generator(device=dev)
    gen.manual_seed(wl.seed + 17)
    bf = torch.bfloat16
    dY = torch.randn(tuple(layer.Y.shape), generator=gen, device=dev).to(bf)
    # the parts' own inputs
    B, H, L = cfg.B, cfg.H, cfg.L
    u8 = dict(dtype=torch.uint8, device=dev)
    status = layer.status
    o_sm = torch.empty((B, L, H, 128), dtype=bf, device=dev)
    lse = torch.empty((B, H, L), dtype=torch.float32, device=dev)
    vdn.vdn_softmax_window_lse(cfg, q, k, v, o_sm, lse,
                               torch.empty(vdn.vdn_workspace_size(cfg, vdn.VDN_WS_SOFTMAX), **u8),
                               status, stream)
    do_sm = torch.randn((B, L, H, 128), generator=gen, device=dev).to(bf)
    do_lin = torch.randn((B, H, L, 128), generator=gen, device=dev).to(bf)
    dq, dk, dv = (torch.empty((B, H, L, 128), dtype=bf, device=dev) for _ in range(3))
    dZ = torch.empty_like(layer.Z)
    dW1 = torch.empty((H * 128, cfg.d_out), dtype=torch.float32, device=dev)
    dW2 = torch.empty_like(dW1)
    sws = torch.empty(vdn.vdn_workspace_size(cfg, vdn.VDN_WS_SOFTMAX_BWD), **u8)
    lws = torch.empty(vdn.vdn_workspace_size(cfg, vdn.VDN_WS_LINEAR_BWD), **u8)
    parts = {
        "merge_bwd": lambda: vdn.vdn_gated_merge_bwd(cfg, layer.Z, W1, W2, dY, dZ, dW1, dW2,
                                                     status, stream),
        "linear_bwd": lambda: vdn.vda_linear_bwd(cfg, q, k, v, do_lin, dq, dk, dv, lws, status,
                                                 stream),
        "softmax_bwd": lambda: vdn.vdn_softmax_window_bwd(cfg, q, k, v, o_sm, lse, do_sm, dq, dk,
                                                          dv, sws, status, stream),
    }

    def check(where):
        st = vdn.vdn_read_status(status, stream)
        if st != 0:
            raise RuntimeError(f"device status {where}: {vdn.vdn_status_string(st)}")

    def timed(fn, n):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
        for i in range(n):
            ev[i].record(stream)
            fn()
        ev[n].record(stream)
        torch.cuda.synchronize(dev)
        return [ev[i].elapsed_time(ev[i + 1]) for i in range(n)]

    for _ in range(args.warmup):
        layer.backward(dY, stream)
    for fn in parts.values():
        fn()
    torch.cuda.synchronize(dev)
    check("after warm-up")
    clocks = ClockSampler(_physical_gpu(local_rank))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    time.sleep(0.3)
    step_ms = float(np.mean(timed(lambda: layer.backward(dY, stream), args.steps)))
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    part_ms = {n: float(np.mean(timed(fn, max(1, min(args.steps, 3))))) for n, fn in parts.items()}
    check("after timing")
    # end to end: a training step from pinned host memory (q, k, v, dY in;
    # every gradient out), forward and backward
    hin = [t.to("cpu").pin_memory() for t in (q, k, v, dY)]
    outs = (layer.dq, layer.dk, layer.dv, layer.dgate, layer.dW1, layer.dW2)
    hout = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs]
    dbuf = [torch.empty_like(t) for t in (q, k, v, dY)]

    def train_step():
        for d_, h_ in zip(dbuf, hin):
            d_.copy_(h_, non_blocking=True)
        layer.forward(dbuf[0], dbuf[1], dbuf[2], gate, W1, W2, stream)
        layer.backward(dbuf[3], stream)
        for h_, d_ in zip(hout, outs):
            h_.copy_(d_, non_blocking=True)

    train_step()
    torch.cuda.synchronize(dev)
    e2e_ms = float(np.mean(timed(train_step, max(1, min(args.steps, args.e2e_steps or 4)))))
    check("after the end-to-end steps")
    step_ms, e2e_ms = max_over_ranks([step_ms, e2e_ms], world, dev)
    if rank != 0:
        return None
    peaks, peak_src = load_peaks()
    flops, _, density = softmax_work(cfg)
    # the softmax backward's algorithmic work: five products per allowed pair
    # (scores again, dP = do v^T, dv = P^T do, dq = dS k, dk = dS^T q), 2.5x the
    # forward's two
    sm_flops = 2.5 * flops
    achieved = sm_flops / (part_ms["softmax_bwd"] * 1e-3) / 1e12
    peak = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
    tokens = cfg.B * cfg.L * world
    kern = {n: {"ms": part_ms[n]} for n in parts}
    kern["softmax_bwd"]["TFLOP/s"] = achieved
    mflops = 2 * (2.0 * cfg.B * cfg.L * 2 * cfg.H * cfg.dv * cfg.d_out)
    kern["merge_bwd"]["TFLOP/s"] = mflops / (part_ms["merge_bwd"] * 1e-3) / 1e12
    return {
        "metric": BWD_METRIC, "value": tokens / (step_ms * 1e-3), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"{wl.name} backward: B={cfg.B} H={cfg.H} d={cfg.d} dv={cfg.dv} "
                               f"T={cfg.T} N={cfg.N} d_out={cfg.d_out}"
                               + (f" n_ctx={cfg.n_ctx}" if cfg.n_ctx else ""),
                   "tokens_per_layer": cfg.B * cfg.L, "mask_density": density,
                   "l2": "inputs larger than L2",
                   "parallelism": f"dp{world}" if world > 1 else "single"},
        "e2e": {"value": tokens / (e2e_ms * 1e-3), "unit": UNIT,
                "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in hin),
                "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in hout),
                "how": "training step from pinned host q, k, v, dY: vdn_hybrid_forward_train "
                       "then vdn_hybrid_backward, every gradient copied back"},
        "gpu_launches": backward_launches(cfg) * args.steps,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": None,
                     "kernel": "softmax_bwd_dkdv_kernel + softmax_bwd_dq_kernel",
                     "peak_source": f"{peak_src} bf16_tflops_sustained",
                     "work": "2.5 x the forward's QK^T + PV FLOPs"},
        "kernels": kern,
        "clocks": clk,
    }


def _e2e(args, inputs, y_like, run, stream, dev, world):
    """End-to-end layer calls from pinned host buffers: every step copies its
    inputs from pinned host memory, runs `run(inputs, Y)` and copies Y back;
    the copies run on their own streams, double-buffered, so that each step's
    copies overlap its neighbours' compute."""
    import torch.distributed as dist

    hin = [t.to("cpu").pin_memory() for t in inputs]
    hY = [torch.empty(y_like.shape, dtype=y_like.dtype).pin_memory() for _ in range(2)]
    # the first step's input copy and the last step's output copy have no
    # neighbour to overlap with; the more steps, the less they weigh
    e2e_steps = max(1, args.e2e_steps or args.steps)
    dq = [tuple(inputs), tuple(torch.empty_like(t) for t in inputs)]
    dY = [y_like, torch.empty_like(y_like)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = {n: [torch.cuda.Event() for _ in range(2)] for n in ("in", "comp", "out")}

    def h2d(i):
        b = i % 2
        s_in.wait_event(ev["comp"][b])        # step i-2 is done with this input set
        with torch.cuda.stream(s_in):
            for dst, src in zip(dq[b], hin):
                dst.copy_(src, non_blocking=True)
        ev["in"][b].record(s_in)

    def e2e_run(n):
        h2d(0)
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                h2d(i + 1)
            stream.wait_event(ev["in"][b])
            stream.wait_event(ev["out"][b])   # step i-2's output copy has read dY[b]
            run(dq[b], dY[b])
            ev["comp"][b].record(stream)
            s_out.wait_event(ev["comp"][b])
            with torch.cuda.stream(s_out):
                hY[b].copy_(dY[b], non_blocking=True)
            ev["out"][b].record(s_out)

    for e in ev["comp"] + ev["out"]:
        e.record(stream)
    e2e_run(2)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    e2e_run(e2e_steps)
    s_out.wait_event(ev["out"][(e2e_steps - 1) % 2])
    e1.record(s_out)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / e2e_steps
    last = (e2e_steps - 1) % 2
    if not torch.equal(hY[last].to(dev), dY[last]):
        raise RuntimeError("end-to-end output differs from its device copy")
    return {"ms": ms, "h2d": sum(t.numel() * t.element_size() for t in hin),
            "d2h": hY[0].numel() * hY[0].element_size()}


def _layer_views(cfg, layer, dev):
    """Split the layer workspace the way vdn_hybrid_forward does."""
    import softmax_attention_video_vdn_b200 as vdn
    a = lambda n: (n + 255) // 256 * 256  # noqa: E731
    frames = cfg.B * cfg.H * cfg.T
    states = cfg.B * cfg.H * cfg.nb * cfg.dv * cfg.d
    sizes = [frames * cfg.d * cfg.d * 4, frames * cfg.dv * cfg.d * 4, states * 4, states * 4,
             cfg.B * cfg.L * 2 * cfg.H * cfg.dv * (2 if cfg.dtype == vdn.VDN_BF16 else 4),
             vdn.vdn_workspace_size(cfg, vdn.VDN_WS_SCAN),
             256]
    views, off = [], 0
    for s in sizes:
        views.append(layer.ws[off:off + s])
        off += a(s)
    G = views[0].view(torch.float32).view(cfg.B, cfg.H, cfg.T, cfg.d, cfg.d)
    C = views[1].view(torch.float32).view(cfg.B, cfg.H, cfg.T, cfg.dv, cfg.d)
    S_fwd = views[2].view(torch.float32).view(cfg.B, cfg.H, cfg.nb, cfg.dv, cfg.d)
    S_bwd = views[3].view(torch.float32).view(cfg.B, cfg.H, cfg.nb, cfg.dv, cfg.d)
    zdt = torch.bfloat16 if cfg.dtype == vdn.VDN_BF16 else torch.float32
    Z = views[4].view(zdt).view(cfg.B, cfg.L, 2, cfg.H, cfg.dv)
    return G, C, S_fwd, S_bwd, Z, views[5], views[6]


# ------------------------------------------------------- CPU oracle sample
def cpu_oracle_sample(wl, x_head, rows, W1, W2, gate):
    """Time the oracle on one head: full linear branch, the softmax of `rows`
    query rows, and the merge of those rows. Returns seconds per part."""
    import oracle as O
    q, k, v = x_head
    t0 = time.perf_counter()
    lb = O.linear_branch(q, k, v, wl.T, wl.N, wl.lam, wl.beta, wl.block_frames,
                         wl.window_blocks, wl.anchors)
    t1 = time.perf_counter()
    mask = O.frame_mask(wl.T, wl.block_frames, wl.window_blocks, wl.anchors)
    osm = O.softmax_window_rows(rows, q, k, v, wl.N, mask, 1.0 / math.sqrt(wl.d))
    t2 = time.perf_counter()
    o_sm = np.broadcast_to(osm[None, None], (1, wl.H, len(rows), wl.dv))
    o_lin = np.broadcast_to(lb["o_lin"][rows][None, None], (1, wl.H, len(rows), wl.dv))
    O.gated_merge(np.ascontiguousarray(o_sm), np.ascontiguousarray(o_lin), gate, W1, W2,
                  wl.w_per_head)
    t3 = time.perf_counter()
    return t1 - t0, t2 - t1, t3 - t2


def cpu_baseline(wl, x, n_rows, seed=0):
    """Oracle throughput extrapolated to the whole layer from a bounded sample:
    one head's full linear branch, n_rows random query rows of that head's
    softmax, and the merge of those rows (all heads' width)."""
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(wl.L, size=n_rows, replace=False))
    head = tuple(x[n][0, 0].double().cpu().numpy() for n in ("q", "k", "v"))
    W1 = x["W1"].double().cpu().numpy()
    W2 = x["W2"].double().cpu().numpy()
    gate = x["gate_logits"].double().cpu().numpy()
    t_lin, t_sm, t_mg = cpu_oracle_sample(wl, head, rows, W1, W2, gate)
    layer_s = wl.H * wl.B * t_lin + (wl.H * wl.B * t_sm + wl.B * t_mg) * wl.L / n_rows
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count()
    sample = (f"1 of {wl.B * wl.H} (b,h): full linear branch ({t_lin:.2f} s), softmax of "
              f"{n_rows} random query rows ({t_sm:.2f} s), merge of those rows ({t_mg:.2f} s); "
              f"extrapolated to the layer ({layer_s:.1f} s)")
    return {"value": wl.B * wl.L / layer_s, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": sample, "sample_s": t_lin + t_sm + t_mg, "layer_s_extrapolated": layer_s}


def run_reference(args, rank, world):
    """The oracle arm: fp64 NumPy on the host cores, bounded samples."""
    if rank != 0:
        return None
    from synthetic import make_inputs
    wl, cfg = workload_cfg(args.workload)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    x = make_inputs(wl, device=dev)
    res = None
    times = []
    for i in range(args.warmup + args.steps):
        r = cpu_baseline(wl, x, args.cpu_rows, seed=i)
        if i >= args.warmup:
            times.append(r["layer_s_extrapolated"])
            res = r
    layer_s = float(np.mean(times))
    value = wl.B * wl.L / layer_s
    res = dict(res, value=value)
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": layer_s * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": workload_name(wl, cfg), "tokens_per_layer": cfg.B * cfg.L},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "cpu_baseline": res,
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--e2e-steps", type=int, default=0,
                    help="end-to-end steps (0: as many as --steps)")
    ap.add_argument("--cpu-rows", type=int, default=512)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--fp8", action="store_true",
                    help="softmax branch on e4m3 q, k, v (per-(b, h) scales)")
    ap.add_argument("--n-ctx", type=int, default=0,
                    help="context (text / audio) tokens after the video tokens of each head")
    ap.add_argument("--ulysses", action="store_true",
                    help="the head-sharded path even at N = 1 (a one-rank process group)")
    ap.add_argument("--dp", action="store_true",
                    help="with --gpus N > 1: N independent replicas of the layer (weak "
                         "scaling) instead of one layer split by heads")
    ap.add_argument("--backward", action="store_true",
                    help="time the layer backward (vdn_hybrid_backward) instead of the forward")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            ap.error("--gpus N > 1 needs torchrun (one process per GPU)")
    head_sharded = (world > 1 or args.ulysses) and not args.dp and not args.backward \
        and args.impl == "ours"
    if args.ulysses and args.dp:
        ap.error("--ulysses and --dp exclude each other")
    dist_init = world > 1 or head_sharded
    if head_sharded and world > 1:
        # NCCL's communicator set-up lines (transport, NVLS or not) on stderr
        os.environ.setdefault("NCCL_DEBUG", "INFO")
        os.environ.setdefault("NCCL_DEBUG_SUBSYS", "INIT")
    if dist_init:
        import datetime

        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", "29517")
        os.environ.setdefault("RANK", str(rank))
        os.environ.setdefault("WORLD_SIZE", str(world))
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local_rank)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))

    if args.impl == "reference":
        res = run_reference(args, rank, world)
    elif args.backward:
        res = run_backward(args, rank, world, local_rank)
    elif head_sharded:
        res = run_ulysses(args, rank, world, local_rank)
    else:
        res = run_ours(args, rank, world, local_rank)
        # the oracle's sampled timing covers video-only sequences
        if res is not None and world == 1 and not args.no_cpu_baseline and not args.n_ctx:
            from synthetic import get_workload, make_inputs
            wl = get_workload(args.workload)
            x = make_inputs(wl, device=torch.device("cuda", local_rank))
            res["cpu_baseline"] = cpu_baseline(wl, x, args.cpu_rows)
            del x
    if dist_init:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0 and res is not None:
        print(json.dumps(res))


if __name__ == "__main__":
    main()
