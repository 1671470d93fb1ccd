#!/usr/bin/env python
"""Benchmark of the spatiotemporal attention hot path on B200.

Default workload (one GPU): Wan2.1-1.3B-like full bidirectional attention
with fused 3D-RoPE, B=1, 12 heads, head dim 128, latent grid 21x30x52
(32760 tokens), bf16 N(0,1) synthetic inputs.  One step = one
vattn_attention call (RoPE fused) on inputs resident in HBM; L2 is flushed
(256 MiB write) before every timed step.  Throughput is mask-adjusted
TFLOP/s: 4 * d FLOPs per visible (query, key) pair per head.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun): every rank runs its own replica of the workload (the
path shards over independent problems; no data-path collective); the time is
the max over ranks and `value` counts the work of all ranks (weak scaling).
--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload on the host cores (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import seeded_inputs as si  # noqa: E402

METRIC = "attention TFLOPS (mask-adjusted) & % of B200 BF16 peak; streaming frames/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = ["video_diffusion_transformer_02_b200/csrc/attention.cuh",
                  "video_diffusion_transformer_02_b200/csrc/attention_pair.cuh",
                  "video_diffusion_transformer_02_b200/csrc/sm100.cuh"]


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def kernel_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per launch of the attention kernel from the committed ncu
    summary, if it was taken on the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "attn_pair_traffic.txt")
    if not os.path.exists(p):
        return None
    vals = {}
    with open(p) as f:
        for line in f:
            if "=" in line and not line.startswith("#"):
                k, v = line.split("=", 1)
                vals[k.strip()] = v.strip()
    if vals.get("kernel_hash") != kernel_hash():
        return None
    try:
        return float(vals["bytes_per_launch_wan13b"])
    except (KeyError, ValueError):
        return None


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples (SM clock, throttle reasons) during the timed region."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if not self.proc:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, parts[3:7]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ------------------------------------------------------------ multi-rank
def reduce_max(value: float, world: int, device=None) -> float:
    """Max over ranks of a per-rank device time (every rank calls it)."""
    if world <= 1:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_step: float, steps: int, world: int, max_total_ms: float) -> float:
    """Whole-job throughput: every rank runs its own replica of the step
    (weak scaling), so the job does world * steps steps in the slowest
    rank's time."""
    return world * flops_per_step * steps / (max_total_ms / 1e3) / 1e12


# -------------------------------------------------------------- workloads
def wan13b_workload(va, torch, device):
    c = si.CONFIGS["wan13b"]
    B, H, d, T, Hg, Wg = c["B"], c["H"], c["d"], c["T"], c["Hg"], c["Wg"]
    L = T * Hg * Wg
    q, k, v = si.qkv("wan13b")
    dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(device)
    rope = va.Rope(Hg=Hg, Wg=Wg, pairs=c["pairs"], max_pos=max(T, Hg, Wg), theta=c["theta"])
    tab = va.rope_table(rope, d, device=device)
    # rotated keys, then the tail split of the last partial wave (zero-filled)
    ws = torch.zeros(va.vattn_attention_workspace_bytes_ex(B, L, L, H, H, d, "full", rope, device=device),
                     dtype=torch.uint8, device=device)
    w = dict(name="wan13b", B=B, H=H, d=d, L=L, T=T, Hg=Hg, Wg=Wg, rope=rope, tab=tab, ws=ws,
             q_host=q, k_host=k, v_host=v, q=dev(q), k=dev(k), v=dev(v),
             o=torch.empty((B, L, H, d), dtype=torch.bfloat16, device=device),
             flops=4.0 * d * L * L * H * B, scale=d ** -0.5, pairs=c["pairs"], theta=c["theta"])
    return w


def run_ours(args, rank, world, device):
    import torch
    import video_diffusion_transformer_02_b200 as va

    torch.cuda.set_device(device)
    dev_index = torch.cuda.current_device()
    w = wan13b_workload(va, torch, device)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()

    def step():
        va.vattn_attention(w["q"], w["k"], w["v"], w["o"], scale=w["scale"], rope=w["rope"],
                           table=w["tab"], workspace=w["ws"])

    kr = torch.empty_like(w["k"])

    def rope_k_only():   # the key-rotation pass of a step, timed alone for the kernel split
        va.vattn_rope_qk(None, w["k"], None, kr, w["rope"], w["tab"])

    for _ in range(args.warmup):
        step()
    va.vattn_check()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    sampler = ClockSampler(dev_index)
    sampler.start()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    va.vattn_check()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    total_ms = float(sum(step_ms))
    rope_ms = _time_events(torch, rope_k_only, args.steps, flush)
    total_ms = reduce_max(total_ms, world, device)
    ms_per_step = total_ms / args.steps
    value = job_tflops(w["flops"], args.steps, world, total_ms)
    # two launches per step: the key rotation (HBM pass) and the attention
    # kernel; the attention kernel's duration is the step minus the rotation
    # pass timed alone on the same stream
    kernel_ms = statistics.mean(step_ms) - rope_ms
    achieved = w["flops"] / (kernel_ms / 1e3) / 1e12

    # end to end through the C ABI with host buffers: every step copies its
    # q, k, v from pinned host memory to the device, runs the call and reads
    # o back to pinned host memory, all inside the timed region.  Steps are
    # pipelined the way a serving loop runs them: two device buffer sets, the
    # H2D copies on one copy stream and the D2H on another, ordered by CUDA
    # events, so the copies of steps i+1 and i-1 overlap the kernels of step
    # i (bytes per step unchanged).
    qh = torch.from_numpy(w["q_host"].view(np.int16)).view(torch.bfloat16).pin_memory()
    kh = torch.from_numpy(w["k_host"].view(np.int16)).view(torch.bfloat16).pin_memory()
    vh = torch.from_numpy(w["v_host"].view(np.int16)).view(torch.bfloat16).pin_memory()
    oh = torch.empty(w["o"].shape, dtype=torch.bfloat16).pin_memory()
    sets = [tuple(torch.empty_like(w[n]) for n in ("q", "k", "v", "o")) for _ in range(2)]
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_run(n):
        for i in range(n):
            qs, ks, vs, os_ = sets[i % 2]
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(ev_out[i % 2])    # step i-2 has finished with this set
                qs.copy_(qh, non_blocking=True)
                ks.copy_(kh, non_blocking=True)
                vs.copy_(vh, non_blocking=True)
                ev_in[i % 2].record(up)
            stream.wait_event(ev_in[i % 2])
            va.vattn_attention(qs, ks, vs, os_, scale=w["scale"], rope=w["rope"], table=w["tab"],
                               workspace=w["ws"])
            ev_done[i % 2].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(ev_done[i % 2])
                oh.copy_(os_, non_blocking=True)
                ev_out[i % 2].record(down)
        stream.wait_event(ev_out[(n - 1) % 2])

    e2e_run(2)
    torch.cuda.synchronize()
    e_steps = max(2, min(args.steps, 10))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    up.wait_event(e0)
    e2e_run(e_steps)
    e1.record(stream)
    torch.cuda.synchronize()
    va.vattn_check()
    e2e_ms = e0.elapsed_time(e1) / e_steps
    e2e_ms = reduce_max(e2e_ms, world, device)
    e2e_exact = bool(torch.equal(oh, w["o"].cpu()))   # same inputs as the device-resident steps
    h2d = 3 * w["q"].numel() * 2
    d2h = w["o"].numel() * 2
    del sets

    secondary = None
    if not args.no_secondary and rank == 0:
        secondary = secondary_measurements(va, torch, device, flush)

    pk, src = peaks()
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, rows=args.cpu_rows)
    return dict(
        metric=METRIC, value=value, unit="TFLOP/s", n_gpus=world, steps=args.steps,
        warmup=args.warmup, ms_per_step=ms_per_step, higher_is_better=True, scaling="weak",
        vs_baseline=None, dtype="bf16", data="synthetic",
        config=workload_config(w["flops"], world),
        roofline={"bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"],
                  "unit": "TFLOP/s", "frac": achieved / pk["bf16_tflops"],
                  "frac_of_sustained": achieved / pk.get("bf16_tflops_sustained", pk["bf16_tflops"]),
                  "peak_source": src + " (burst bf16 GEMM)", "kernel": "attn_pair_kernel<128,rope-q>",
                  "kernel_ms": kernel_ms, "rope_k_ms": rope_ms, "traffic": recorded_traffic()},
        cpu_baseline=cpu,
        e2e={"value": w["flops"] / (e2e_ms / 1e3) / 1e12 * world, "unit": "TFLOP/s",
             "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
             "steps": e_steps, "pipelined": "two buffer sets; H2D of step i+1 and D2H of step i-1 overlap step i",
             "output_equals_device_step": e2e_exact},
        clocks=clocks, gpu_launches=2 * args.steps, secondary=secondary)


def _time_events(torch, fn, n, flush=None):
    """Mean ms of n runs of fn, each bracketed by CUDA events on the current
    stream (L2 flushed before each run, outside the events, when given)."""
    return statistics.mean(_event_list(torch, fn, n, flush))


def _event_list(torch, fn, n, flush=None):
    s = torch.cuda.current_stream()
    out = []
    for _ in range(n):
        if flush is not None:
            flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s)
        fn()
        b.record(s)
        torch.cuda.synchronize()
        out.append(a.elapsed_time(b))
    return out


REPS = 20   # timed repetitions of every secondary figure (median reported)


def _measure(torch, fn, reps=REPS, flush=None, per_call=1):
    """Median of `reps` event-timed runs of fn (after one untimed run), with
    the nvidia-smi clock record of the timed runs.  per_call: calls of the
    measured operation inside one run of fn (the figure is per call)."""
    fn()
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    ms = _event_list(torch, fn, reps, flush)
    clocks = sampler.stop()
    ms = [m / per_call for m in ms]
    return {"median_ms": statistics.median(ms), "min_ms": min(ms), "max_ms": max(ms), "reps": reps,
            "clocks": clocks}


def _graph(torch, calls):
    """A CUDA graph replaying `calls` (a list of callables) back to back."""
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        calls[0]()
        with torch.cuda.graph(g, stream=side):
            for c in calls:
                c()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    return g


def _hbm(pk, nbytes, m):
    gbs = nbytes / (m["median_ms"] / 1e3) / 1e9
    return {"bytes": nbytes, "us": m["median_ms"] * 1e3, "gbs": gbs, "frac_of_hbm": gbs / pk["hbm_gbs"]}


def secondary_measurements(va, torch, device, flush):
    """The other configurations: 14B full / chunk-causal TFLOPS, streaming
    frames/s and its fraction of the tensor-peak ceiling, the KV append, the
    hybrid call and its state delta and scan kernels (GB/s, fraction of HBM).
    Every figure is the median of REPS event-timed runs with its own clock
    record."""
    out = {}
    dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(device)
    pk, _ = peaks()
    # Wan2.1-14B-like 720p
    c = si.CONFIGS["wan14b"]
    L, H, d = c["T"] * c["Hg"] * c["Wg"], c["H"], c["d"]
    q, k, v = si.qkv("wan14b")
    qd, kd, vd = dev(q), dev(k), dev(v)
    del q, k, v
    o = torch.empty_like(qd)
    rope = va.Rope(Hg=c["Hg"], Wg=c["Wg"], pairs=c["pairs"], max_pos=max(c["T"], c["Hg"], c["Wg"]))
    tab = va.rope_table(rope, d, device=device)
    F = c["Hg"] * c["Wg"]
    ws14 = torch.empty(va.vattn_attention_workspace_bytes(1, L, H, d, rope), dtype=torch.uint8, device=device)
    for name, mode, frac in (("wan14b_full", "full", 1.0), ("wan14b_chunk", "chunk_causal", 28 / 49)):
        fn = lambda: va.vattn_attention(qd, kd, vd, o, scale=d ** -0.5, mode=mode, tokens_per_frame=F,
                                        chunk_frames=c["chunk_frames"], rope=rope, table=tab, workspace=ws14)
        m = _measure(torch, fn)          # inputs 2.3 GB: far larger than L2
        flops = 4.0 * d * L * L * H * frac
        tf = flops / m["median_ms"] * 1e-9
        out[name] = dict(m, tflops=tf, frac_of_peak=tf / pk["bf16_tflops"], mask_adjusted_flops=flops)
    del qd, kd, vd, o, ws14
    # streaming decode: 32 frames, ring of 4, window 4
    c = si.CONFIGS["stream"]
    F, H, d, T = c["Hg"] * c["Wg"], c["H"], c["d"], c["T"]
    q, k, v = si.qkv("stream")
    qd, kd, vd = dev(q).view(T, F, H, d), dev(k).view(T, F, H, d), dev(v).view(T, F, H, d)
    cap = c["capacity"]
    kr = torch.zeros((cap, 1, F, H, d), dtype=torch.bfloat16, device=device)
    vr = torch.zeros_like(kr)
    ids = torch.zeros(cap, dtype=torch.int32, device=device)
    cache = va.KVCache(kr, vr, ids)
    rope = va.Rope(Hg=c["Hg"], Wg=c["Wg"], pairs=c["pairs"], max_pos=64)
    tab = va.rope_table(rope, d, device=device)
    cache.enable_rope(torch.zeros((cap + 1, 1, F, H, d), dtype=torch.bfloat16, device=device), rope, tab)
    of = torch.empty((1, F, H, d), dtype=torch.bfloat16, device=device)
    frames = [(qd[f].unsqueeze(0), kd[f].unsqueeze(0), vd[f].unsqueeze(0)) for f in range(T)]

    def stream_all():
        for f in range(T):
            qf, kf, vf = frames[f]
            cache.attend(qf, kf, vf, of, f, c["window_back"], rope=rope, table=tab)
            cache.append(kf, vf, f)

    m = _measure(torch, stream_all)
    pairs_frames = sum(min(f, c["window_back"]) + 1 for f in range(T))   # (q-frame, k-frame) pairs: 150
    total_flops = 4.0 * d * F * F * H * pairs_frames
    tf = total_flops / m["median_ms"] * 1e-9
    fps = T / (m["median_ms"] / 1e3)
    # ceiling: the whole 32-frame stream's mask-adjusted FLOPs at the
    # measured bf16 peak; frames/s over the ceiling = TFLOP/s over the peak
    ceiling_fps = T / (total_flops / (pk["bf16_tflops"] * 1e12))
    steady_flops = 4.0 * d * F * F * H * (c["window_back"] + 1)
    stream = dict(m, frames_per_s=fps, ms_per_frame=m["median_ms"] / T, tflops=tf,
                  frac_of_ceiling=fps / ceiling_fps, ceiling_frames_per_s=ceiling_fps,
                  ceiling_steady_frames_per_s=pk["bf16_tflops"] * 1e12 / steady_flops,
                  ceiling_formula="frames/s at the measured bf16 peak = T * peak / (4 d F^2 H * 150); "
                                  "150 = visible (query frame, key frame) pairs of the 32-frame stream")
    steady = lambda: cache.attend(frames[10][0], frames[10][1], frames[10][2], of, T - 1,
                                  c["window_back"], rope=rope, table=tab)
    ms_ = _measure(torch, steady)
    stream["steady_attention"] = dict(ms_, tflops=steady_flops / ms_["median_ms"] * 1e-9,
                                      frac_of_peak=steady_flops / ms_["median_ms"] * 1e-9 / pk["bf16_tflops"])
    # KV append of one frame: a single launch after an L2 flush, and 16
    # appends of distinct frames (inputs 134 MB, more than L2) replayed from
    # a CUDA graph.  In the streaming loop the append after attend is a
    # plain copy (the attend call already rotated the frame's keys): read k,
    # v; write raw k, v.  An append without a preceding attend also writes
    # the rotated keys.
    app_bytes = 4 * F * H * d * 2
    rot_bytes = 5 * F * H * d * 2
    plain = va.KVCache(torch.zeros_like(kr), torch.zeros_like(vr), torch.zeros_like(ids))
    one = _measure(torch, lambda: plain.append(frames[3][1], frames[3][2], 3), flush=flush)
    g = _graph(torch, [lambda f=f: plain.append(frames[f][1], frames[f][2], f) for f in range(16)])
    batch = _measure(torch, g.replay, per_call=16)
    del g
    plain.close()
    g = _graph(torch, [lambda f=f: cache.append(frames[f][1], frames[f][2], f) for f in range(16)])
    batch_rot = _measure(torch, g.replay, per_call=16)
    del g
    stream["append"] = {"single_launch": _hbm(pk, app_bytes, one), "graph16": _hbm(pk, app_bytes, batch),
                        "rotated_graph16": _hbm(pk, rot_bytes, batch_rot),
                        "clocks": batch["clocks"]}
    out["stream"] = stream
    cache.close()
    del kr, vr
    # the same stream through the one-launch step (attend + append fused),
    # ring of W + 1 = 5 frames
    out["stream_step"] = stream_step_figure(va, torch, device, frames, c, pk, window_relative=False)
    del qd, kd, vd, frames
    # FlashDecoder-XL-shaped streams: 24 heads on 3 KV heads, window 2,
    # positions relative to the window, one launch per step
    for name in ("xl480", "xl720", "xl480_refine"):
        cx = si.CONFIGS[name]
        Fx = cx["sub"] * cx["Hg"] * cx["Wg"]
        qx, kx, vx = si.qkv(name)
        Tx = cx["T"]
        qd = dev(qx).view(Tx, Fx, cx["H"], cx["d"])
        kd = dev(kx).view(Tx, Fx, cx["Hkv"], cx["d"])
        vd = dev(vx).view(Tx, Fx, cx["Hkv"], cx["d"])
        fr = [(qd[f].unsqueeze(0), kd[f].unsqueeze(0), vd[f].unsqueeze(0)) for f in range(Tx)]
        out[name] = stream_step_figure(va, torch, device, fr, cx, pk, window_relative=True)
        del qd, kd, vd, fr
    # hybrid chunk attention
    c = si.CONFIGS["hybrid"]
    L, H, d = c["T"] * c["Hg"] * c["Wg"], c["H"], c["d"]
    ct = c["chunk_frames"] * c["Hg"] * c["Wg"]
    q, k, v = si.qkv("hybrid")
    qd, kd, vd = dev(q), dev(k), dev(v)
    o = torch.empty_like(qd)
    S = torch.zeros((1, H, d, d), dtype=torch.float32, device=device)
    z = torch.zeros((1, H, d), dtype=torch.float32, device=device)
    wsb = va.vattn_hybrid_workspace_bytes(1, L, H, d, ct)
    ws = torch.empty(wsb, dtype=torch.uint8, device=device)
    fn = lambda: va.vattn_hybrid_chunk(qd, kd, vd, o, S, z, ct, workspace=ws)
    m = _measure(torch, fn)
    n_ch = (L + ct - 1) // ct
    intra = sum(min(ct, L - i * ct) ** 2 for i in range(n_ch))
    # softmax part: 4 d per (query, key) pair in the same chunk; state: the
    # build phi(k) v^T + sum phi(k) (2 d^2 + 2 d per key, as multiply-adds)
    # and the read-out phi(q)^T S + phi(q) . z (2 d^2 + 2 d per query)
    flops = 4.0 * d * intra * H + (2.0 * d * d + 2.0 * d) * L * H * 2
    tf = flops / m["median_ms"] * 1e-9
    hyb = dict(m, tflops=tf, frac_of_peak=tf / pk["bf16_tflops"], mask_adjusted_flops=flops,
               flop_formula="4 d sum_c |c|^2 H + (2 d^2 + 2 d) L H (keys) + (2 d^2 + 2 d) L H (queries)")
    # state delta: reads K and V, writes the per-chunk deltas
    delta_bytes = 2 * L * H * d * 2 + wsb
    kd2, vd2 = kd.clone(), vd.clone()      # a second input set: 2 x 149 MB > L2
    one = _measure(torch, lambda: va.vattn_hybrid_delta(kd, vd, ct, ws), flush=flush)
    g = _graph(torch, [lambda i=i: va.vattn_hybrid_delta(kd if i % 2 == 0 else kd2, vd if i % 2 == 0 else vd2,
                                                          ct, ws) for i in range(16)])
    batch = _measure(torch, g.replay, per_call=16)
    del g
    hyb["delta"] = {"single_launch": _hbm(pk, delta_bytes, one), "graph16": _hbm(pk, delta_bytes, batch)}
    # scan: reads and writes the workspace (in place) and the state in/out;
    # the graph cycles over 12 workspaces (209 MB, more than L2)
    scan_bytes = 2 * wsb + 2 * (S.numel() + z.numel()) * 4
    va.vattn_hybrid_delta(kd, vd, ct, ws)
    one = _measure(torch, lambda: va.vattn_hybrid_scan(S, z, L, ct, ws), flush=flush)
    wss = [torch.zeros(wsb, dtype=torch.uint8, device=device) for _ in range(12)]
    g = _graph(torch, [lambda i=i: va.vattn_hybrid_scan(S, z, L, ct, wss[i % 12]) for i in range(16)])
    batch = _measure(torch, g.replay, per_call=16)
    del g, wss
    hyb["scan"] = {"single_launch": _hbm(pk, scan_bytes, one), "graph16": _hbm(pk, scan_bytes, batch)}
    out["hybrid"] = hyb
    # the MobileWan page variant on the same inputs: chunks of 4 frames
    # overlapping 2 frames, polynomial feature maps
    cp = si.CONFIGS["hybrid_page"]
    ctp = cp["chunk_frames"] * cp["Hg"] * cp["Wg"]
    ovp = cp["overlap_frames"] * cp["Hg"] * cp["Wg"]
    coef = torch.from_numpy(si.poly_coef(cp["coef_seed"], H).astype(np.float32)).to(device)
    wsp = torch.empty(va.vattn_hybrid_workspace_bytes_ex(1, L, H, d, ctp, ovp), dtype=torch.uint8, device=device)
    fn = lambda: va.vattn_hybrid_chunk_ex(qd, kd, vd, o, S, z, ctp, ovp, coef=coef, workspace=wsp)
    m = _measure(torch, fn)
    pairs = 0
    for ci in range((L + ctp - 1) // ctp):
        q0, q1 = ci * ctp, min(L, (ci + 1) * ctp)
        pairs += (q1 - q0) * (q1 - max(0, q0 - ovp))
    flops = 4.0 * d * pairs * H + (2.0 * d * d + 2.0 * d) * L * H * 2
    tf = flops / m["median_ms"] * 1e-9
    out["hybrid_page"] = dict(m, tflops=tf, frac_of_peak=tf / pk["bf16_tflops"], mask_adjusted_flops=flops)
    va.vattn_check()
    return out


def stream_step_figure(va, torch, device, frames, c, pk, window_relative):
    """Frames/s of a whole stream decoded with vattn_kvcache_step (attend and
    append in one launch per frame), ring of W + 1 frames, with its fraction
    of the tensor-peak ceiling (the stream's mask-adjusted FLOPs at the
    measured bf16 peak)."""
    T = len(frames)
    _, F, H, d = frames[0][0].shape
    Hkv = frames[0][1].shape[2]
    wb = c["window_back"]
    cap = wb + 1
    kr = torch.zeros((cap, 1, F, Hkv, d), dtype=torch.bfloat16, device=device)
    cache = va.KVCache(kr, torch.zeros_like(kr), torch.zeros(cap, dtype=torch.int32, device=device))
    sub = c.get("sub", 1)
    rope = va.Rope(Hg=c["Hg"], Wg=c["Wg"], pairs=c["pairs"], max_pos=max(64, c["Hg"], c["Wg"]))
    tab = va.rope_table(rope, d, device=device)
    cache.enable_rope(torch.zeros((cap + 1, 1, F, Hkv, d), dtype=torch.bfloat16, device=device), rope, tab)
    of = torch.empty((1, F, H, d), dtype=torch.bfloat16, device=device)
    ws = cache.step_workspace(H, wb)

    def run():
        for f in range(T):
            qf, kf, vf = frames[f]
            cache.step(qf, kf, vf, of, f, wb, rope=rope, table=tab, window_relative=window_relative, workspace=ws)

    m = _measure(torch, run)
    va.vattn_check()
    # the same T steps captured once in a CUDA graph and replayed (the
    # per-frame work is fixed, FlashDecoder "Inference Optimization", Sec.
    # 4.6): no host work between the launches
    g = _graph(torch, [run])
    mg = _measure(torch, g.replay)
    del g
    va.vattn_check()
    cache.close()
    pairs = sum(min(f, wb) + 1 for f in range(T))
    flops = 4.0 * d * F * F * H * pairs
    tf = flops / m["median_ms"] * 1e-9
    fps = T / (m["median_ms"] / 1e3)
    ceiling = T / (flops / (pk["bf16_tflops"] * 1e12))
    fps_g = T / (mg["median_ms"] / 1e3)
    m["graph"] = dict(mg, frames_per_s=fps_g, latent_frames_per_s=fps_g * sub, ms_per_frame=mg["median_ms"] / T,
                      tflops=flops / mg["median_ms"] * 1e-9, frac_of_ceiling=fps_g / ceiling)
    return dict(m, frames_per_s=fps, latent_frames_per_s=fps * sub, ms_per_frame=m["median_ms"] / T, tflops=tf,
                frac_of_ceiling=fps / ceiling, ceiling_frames_per_s=ceiling, launches_per_frame=1,
                workload="%d steps of %d tokens (%d latent frames of %dx%d), H=%d on %d KV heads, d=%d, "
                         "window %d, %s positions" % (T, F, sub, c["Hg"], c["Wg"], H, Hkv, d, wb + 1,
                                                     "window-relative" if window_relative else "absolute"))


def cpu_baseline(w, rows=20480, configs=True):
    """The fp64 oracle, as it stands, on a bounded sample of the workload;
    with `configs`, also the oracle's own timings of the other configurations
    (tiny and hybrid whole, the stream on sampled rows with a projection)."""
    import oracle
    rows_arr = si.sample_rows(0xBA5E, rows, w["B"], 2, w["L"])
    t0 = time.perf_counter()
    oracle.attention(w["q_host"], w["k_host"], w["v_host"], w["scale"],
                     rope=dict(Hg=w["Hg"], Wg=w["Wg"], pairs=w["pairs"], theta=w["theta"]), rows=rows_arr)
    dt = time.perf_counter() - t0
    flops = 4.0 * w["d"] * w["L"] * len(rows_arr)
    out = {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
           "seconds": dt,
           "sample": "%d query rows (2 of 12 heads) of the wan13b workload, all 32760 keys each, "
                     "fp64 with 3D-RoPE; TFLOP/s of mask-adjusted work" % len(rows_arr)}
    if configs:
        out["configs"] = oracle_config_timings(w, len(rows_arr), dt)
    return out


def oracle_config_timings(w, wan_rows, wan_seconds, stream_rows=1024):
    """Host timings of the fp64 oracle per configuration: tiny and hybrid in
    full, the stream and the 1.3B-like workload on sampled query rows with
    the full time projected from rows/s (labelled as a projection)."""
    import oracle
    res = {}
    wan_rps = wan_rows / wan_seconds
    res["wan13b"] = {"rows_sampled": wan_rows, "seconds": wan_seconds, "rows_per_s": wan_rps,
                     "projected_full_s": w["L"] * w["H"] * w["B"] / wan_rps, "projected": True}
    c = si.CONFIGS["tiny"]
    q, k, v = si.qkv("tiny")
    t0 = time.perf_counter()
    oracle.attention(q, k, v, c["d"] ** -0.5, rope=dict(Hg=c["Hg"], Wg=c["Wg"], pairs=c["pairs"], theta=c["theta"]))
    res["tiny"] = {"rows": int(q.shape[1] * q.shape[2]), "seconds": time.perf_counter() - t0, "projected": False}
    c = si.CONFIGS["hybrid"]
    q, k, v = si.qkv("hybrid")
    ct = c["chunk_frames"] * c["Hg"] * c["Wg"]
    t0 = time.perf_counter()
    oracle.hybrid_recurrent(q, k, v, ct, c["d"] ** -0.5)
    res["hybrid"] = {"rows": int(q.shape[1] * q.shape[2]), "seconds": time.perf_counter() - t0, "projected": False}
    del q, k, v
    c = si.CONFIGS["stream"]
    F = c["Hg"] * c["Wg"]
    q, k, v = si.qkv("stream")
    L = q.shape[1]
    srows = si.sample_rows(0x57A, stream_rows, 1, c["H"], L)
    t0 = time.perf_counter()
    oracle.stream(q, k, v, F, c["d"] ** -0.5, c["window_back"],
                  rope=dict(Hg=c["Hg"], Wg=c["Wg"], pairs=c["pairs"], theta=c["theta"]), rows=srows)
    dt = time.perf_counter() - t0
    rps = len(srows) / dt
    res["stream"] = {"rows_sampled": int(len(srows)), "seconds": dt, "rows_per_s": rps,
                     "projected_full_s": L * c["H"] / rps, "projected": True}
    del q, k, v
    return res


def workload_config(flops, world):
    """The benchmarked workload, named the same way by both arms."""
    return {"workload": "wan13b full bidirectional attention + fused 3D-RoPE "
                        "(B=1, H=12, d=128, grid 21x30x52 = 32760 tokens, pairs t22/h21/w21, theta 1e4)",
            "mask_adjusted_flops_per_step": flops,
            "l2": "flushed before every timed step (256 MiB write); inputs 300 MB > L2",
            "parallelism": "replicas x%d" % world}


def run_reference(args, rank, world):
    """The oracle timed on the host as the reference arm (rank 0 only)."""
    if rank != 0:
        return None
    import oracle
    c = si.CONFIGS["wan13b"]
    q, k, v = si.qkv("wan13b")
    L, d = c["T"] * c["Hg"] * c["Wg"], c["d"]
    rope = dict(Hg=c["Hg"], Wg=c["Wg"], pairs=c["pairs"], theta=c["theta"])
    n = args.ref_rows

    def one(i):
        rows = si.sample_rows(0xBA5E + i, n, 1, 2, L)
        oracle.attention(q, k, v, d ** -0.5, rope=rope, rows=rows)
        return len(rows)

    for i in range(args.warmup):
        one(i)
    t0 = time.perf_counter()
    total_rows = 0
    for i in range(args.steps):
        total_rows += one(100 + i)
    dt = time.perf_counter() - t0
    flops = 4.0 * d * L * total_rows
    val = flops / dt / 1e12
    sample = "%d query rows per step (2 of 12 heads) of the wan13b workload, all 32760 keys, fp64" % n
    return dict(metric=METRIC, value=val, unit="TFLOP/s", n_gpus=world, steps=args.steps,
                warmup=args.warmup, ms_per_step=dt / args.steps * 1e3, higher_is_better=True,
                scaling="weak", vs_baseline=None, dtype="f64", data="synthetic", impl="reference",
                config=workload_config(4.0 * d * L * L * c["H"], world),
                cpu_baseline={"value": val, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                              "kind": "oracle", "sample": sample},
                e2e={"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0})


def run_case(args, device):
    """One workload's calls, `steps` times after `warmup`, for profilers (ncu
    captures one kernel of one case): prints one line with the mean time."""
    import torch
    import video_diffusion_transformer_02_b200 as va
    torch.cuda.set_device(device)
    dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(device)
    name = args.case
    if name in ("stream_frame", "xl480_frame", "xl720_frame"):
        cname = {"stream_frame": "stream", "xl480_frame": "xl480", "xl720_frame": "xl720"}[name]
        c = si.CONFIGS[cname]
        F, H, d, wb = c["Hg"] * c["Wg"], c["H"], c["d"], c["window_back"]
        Hkv = c.get("Hkv", H)
        nf = wb + 1
        q, k, v = si.qkv(cname, L=nf * F)
        qd, kd, vd = dev(q).view(nf, F, H, d), dev(k).view(nf, F, Hkv, d), dev(v).view(nf, F, Hkv, d)
        cap = wb + 1
        kr = torch.zeros((cap, 1, F, Hkv, d), dtype=torch.bfloat16, device=device)
        cache = va.KVCache(kr, torch.zeros_like(kr), torch.zeros(cap, dtype=torch.int32, device=device))
        rope = va.Rope(Hg=c["Hg"], Wg=c["Wg"], pairs=c["pairs"], max_pos=4096)   # frame index grows per call
        tab = va.rope_table(rope, d, device=device)
        cache.enable_rope(torch.zeros((cap + 1, 1, F, Hkv, d), dtype=torch.bfloat16, device=device), rope, tab)
        of = torch.empty((1, F, H, d), dtype=torch.bfloat16, device=device)
        rel = cname != "stream"
        for f in range(wb):   # fill the window
            cache.step(qd[f:f + 1], kd[f:f + 1], vd[f:f + 1], of, f, wb, rope=rope, table=tab, window_relative=rel)
        i = [wb]

        def fn():   # one steady frame (the window full), the frame index advancing
            f = i[0]
            cache.step(qd[wb:wb + 1], kd[wb:wb + 1], vd[wb:wb + 1], of, f, wb, rope=rope, table=tab,
                       window_relative=rel)
            i[0] += 1
    elif name in ("hybrid", "hybrid_page"):
        c = si.CONFIGS[name]
        L, H, d = c["T"] * c["Hg"] * c["Wg"], c["H"], c["d"]
        ct = c["chunk_frames"] * c["Hg"] * c["Wg"]
        ov = c.get("overlap_frames", 0) * c["Hg"] * c["Wg"]
        q, k, v = si.qkv(name)
        qd, kd, vd = dev(q), dev(k), dev(v)
        o = torch.empty_like(qd)
        S = torch.zeros((1, H, d, d), dtype=torch.float32, device=device)
        z = torch.zeros((1, H, d), dtype=torch.float32, device=device)
        coef = (torch.from_numpy(si.poly_coef(c["coef_seed"], H).astype(np.float32)).to(device)
                if "coef_seed" in c else None)
        fn = lambda: va.vattn_hybrid_chunk_ex(qd, kd, vd, o, S, z, ct, ov, coef=coef)
    elif name == "wan13b":
        w = wan13b_workload(va, torch, device)
        fn = lambda: va.vattn_attention(w["q"], w["k"], w["v"], w["o"], scale=w["scale"], rope=w["rope"],
                                        table=w["tab"], workspace=w["ws"])
    else:
        raise SystemExit("unknown case %s" % name)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    ms = _event_list(torch, fn, args.steps)
    va.vattn_check()
    print(json.dumps({"case": name, "steps": args.steps, "mean_ms": statistics.mean(ms), "ms": ms}), flush=True)


CASES = ("wan13b", "stream_frame", "xl480_frame", "xl720_frame", "hybrid", "hybrid_page")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=20480)
    ap.add_argument("--ref-rows", type=int, default=512)
    ap.add_argument("--case", choices=CASES, default=None,
                    help="run only this workload's calls (for profilers); prints its mean time")
    args = ap.parse_args()
    if args.case:
        import torch
        run_case(args, torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0"))))
        return
    args.warmup = max(args.warmup, 3) if args.impl == "ours" else args.warmup

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    import torch
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    res = run_ours(args, rank, world, torch.device("cuda", local))
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
