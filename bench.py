#!/usr/bin/env python
"""Throughput of the speech front end + 32-layer ASR encoder on B200: audio seconds encoded
per second, with the dominant kernel's roofline, an end-to-end number through the C-ABI
with host buffers, and the fp64 oracle timed on the host cores.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl sal|reference]

One step = sal_frontend + sal_stack_project + sal_encoder_forward over one batch of the
workload's synthetic audio, inputs resident in HBM, replayed as one CUDA graph. Between
timed steps a 256 MiB buffer (twice the 126 MB L2) is rewritten, outside the timed events.
For N > 1 (torchrun), every rank encodes its own copy of the workload (clips are
independent; no collective on the data path) and the job's time is the max over ranks.
Prints ONE JSON line on rank 0.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from speech_audio_encoder_b200 import synth  # noqa: E402

METRIC = "audio-sec encoded/sec (frontend+32-layer encoder, bf16) on 1 B200; % TC peak"
UNIT = "audio-s/s"
DEFAULT_WORKLOAD = "rec_1h"  # the largest single-GPU configuration
FLUSH_BYTES = 256 << 20

GEMM_FLOPS_PER_POS_LAYER = 2 * (4 * 1280 * 1280 + 2 * 1280 * 5120)  # 39,321,600
STACK_PROJ_FLOPS_PER_POS = 2 * 1024 * 1280
ATTN_FLOPS_PER_T2_LAYER = 4 * 1280  # QK^T and PV over all heads: 4 T^2 * width


def positions(n_samples: int) -> int:
    f = 0 if n_samples < 400 else 1 + (n_samples - 400) // 160
    return f // 8


def frames(n_samples: int) -> int:
    return 0 if n_samples < 400 else 1 + (n_samples - 400) // 160


def attention_pairs(T: int, chunk: int = 0) -> int:
    """Query-key pairs of one clip: T^2, or the sum of squared chunk lengths when attention
    stays inside chunks of ``chunk`` positions."""
    if chunk <= 0 or chunk >= T:
        return T * T
    full, rest = divmod(T, chunk)
    return full * chunk * chunk + rest * rest


def window_lengths(T: int, core: int, context: int) -> list[int]:
    """Positions of each serving window of a clip of T positions: its core of ``core``
    positions (the last may be shorter) and up to ``context`` more on each side."""
    return [min(T, c0 + core + context) - max(0, c0 - context) for c0 in range(0, T, core)]


def layer_work(T: int, chunk: int = 0, window: tuple[int, int] | None = None) -> tuple[int, int]:
    """(positions a layer processes, query-key pairs of its attention) per clip: T and T^2
    (or the sum of squared chunk lengths); with serving windows every window's own
    positions and pairs, context positions included (they are encoded once per window)."""
    if window:
        lens = window_lengths(T, *window)
        return sum(lens), sum(n * n for n in lens)
    return T, attention_pairs(T, chunk)


def kernel_flops(kind: str, B: int, T: int, chunk: int = 0, window=None) -> float:
    """Algorithmic flops of ONE launch of a kernel kind (all clips of the batch)."""
    rows, pairs = layer_work(T, chunk, window)
    M = B * rows
    return {
        "qkv": 2.0 * M * 1280 * 3840,
        "out_proj": 2.0 * M * 1280 * 1280,
        "ffn_up": 2.0 * M * 1280 * 5120,
        "ffn_down": 2.0 * M * 5120 * 1280,
        "attention": float(ATTN_FLOPS_PER_T2_LAYER) * pairs * B,
    }.get(kind, 0.0)


def kernel_bytes(kind: str, B: int, T: int) -> float:
    """Algorithmic HBM bytes of ONE launch of a memory-bound kernel kind."""
    M = B * T
    return {
        "layernorm": M * 1280 * (4 + 2) + 2 * 1280 * 2,
        "rope_table": T * 64 * 2 * 4,
    }.get(kind, 0.0)


def frontend_bytes(B: int, N: int) -> float:
    """Algorithmic HBM bytes of the front end over B clips of N samples: the samples read
    once, the fp32 log-mel [F, 128] and the bf16 stack [T, 1024] written once."""
    F = 0 if N < 400 else 1 + (N - 400) // 160
    T = F // 8
    return float(B) * (4 * N + 512 * F + 2048 * T)


def workload_flops(B: int, T: int, L: int, chunk: int = 0, window=None) -> float:
    rows, pairs = layer_work(T, chunk, window)
    return (GEMM_FLOPS_PER_POS_LAYER * B * rows * L + ATTN_FLOPS_PER_T2_LAYER * pairs * B * L
            + STACK_PROJ_FLOPS_PER_POS * B * T)


# ----------------------------------------------------------------------------- distributed

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(value: float, device=None) -> float:
    """Max of a float over all ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(audio_seconds_per_rank: float, n_ranks: int, max_seconds: float) -> float:
    """Whole-job audio seconds per second: every rank's audio over the slowest rank's time."""
    return audio_seconds_per_rank * n_ranks / max_seconds


def rank_seed_offset(rank: int) -> int:
    """Each rank encodes its own clips: audio seeds are offset by 1000 per rank."""
    return 1000 * rank


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", self.gpu_id],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, power, reasons = [], [], [], set()
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for name, v in zip(self.REASONS, f[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": sorted(reasons), "samples": 0}
        # samples under load: power above the midpoint of the observed range
        pmid = (min(power) + max(power)) / 2
        loaded = [s for s, p in zip(sm, power) if p >= pmid] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm), "power_w_max": max(power)}


# ----------------------------------------------------------------------------- oracle timing

def oracle_step_estimate(wl: synth.Workload, budget_s: float, audio: np.ndarray,
                         weights_f32: dict | None = None):
    """Time the fp64 oracle on a bounded sample of one step and extrapolate to the whole step.

    The sample: the front end on up to ``fe_frames`` frames of one clip; one encoder layer on a
    sub-clip of ``Ts`` positions, repeated while the budget lasts (attention timed apart, so the
    linear part scales with positions and the attention part with positions squared). Returns
    (estimated seconds per step, description, seconds actually spent, threads used).
    """
    import oracle as O

    threads = O.threads()
    t_start = time.perf_counter()
    F, T, B, L = frames(wl.n_samples), positions(wl.n_samples), wl.batch, wl.n_layers
    fe_frames = max(1, min(F, int(4000 * budget_s)))
    t0 = time.perf_counter()
    O.log_mel(audio, first=0, count=fe_frames)
    t_fe = (time.perf_counter() - t0) * (B * F / fe_frames)
    if weights_f32 is None:
        weights_f32 = synth.weights_f32(synth.make_weights(1))
    lw = weights_f32["layers"][0]
    Ts = max(1, min(T, 374))
    rng = np.random.default_rng(0)
    x = rng.standard_normal((Ts, 1280))
    q = rng.standard_normal((10, Ts, 128))
    t_layer, t_attn, reps = [], [], 0
    while True:
        t0 = time.perf_counter()
        O.encoder_layer(x, lw)
        t_layer.append(time.perf_counter() - t0)
        t0 = time.perf_counter()
        O.attention(q, q, q)
        t_attn.append(time.perf_counter() - t0)
        reps += 1
        if time.perf_counter() - t_start > budget_s:
            break
    tl, ta = float(np.median(t_layer)), float(np.median(t_attn))
    ta = min(ta, tl)
    t_lin = tl - ta
    t_proj = t_lin * (STACK_PROJ_FLOPS_PER_POS / GEMM_FLOPS_PER_POS_LAYER)
    est = t_fe + B * (T / Ts) * (L * t_lin + t_proj) + B * L * ta * (T / Ts) ** 2
    spent = time.perf_counter() - t_start
    desc = (f"front end on {fe_frames} of {F} frames of one clip; one encoder layer on {Ts} of {T} "
            f"positions, {reps} run(s), attention timed apart; scaled to {B} clip(s) x {L} layers "
            f"by flop count")
    return est, desc, spent, threads


# ----------------------------------------------------------------------------- reference arm

def run_reference(args, wl: synth.Workload) -> dict | None:
    world, rank, _ = dist_env()
    if rank != 0:
        return None
    budget = max(0.05, 120.0 / max(1, args.steps + args.warmup))
    wf = synth.weights_f32(synth.make_weights(1))
    audio = synth.Workload(wl.name, 1, wl.n_samples, wl.n_layers, wl.kind, wl.seed).audio()[0]
    for _ in range(args.warmup):
        oracle_step_estimate(wl, budget, audio, wf)
    ests, spent_total, desc, threads = [], 0.0, "", 1
    for _ in range(args.steps):
        est, desc, spent, threads = oracle_step_estimate(wl, budget, audio, wf)
        ests.append(est)
        spent_total += spent
    sec = float(np.mean(ests))
    value = wl.audio_seconds / sec
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": wl.name, "batch": wl.batch, "n_samples": wl.n_samples,
                   "positions": positions(wl.n_samples), "layers": wl.n_layers,
                   "parallelism": "host cores, rank 0 only"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "cpu_model": _cpu_model(), "nproc": os.cpu_count(),
                         "sample": desc + f"; {args.steps} samples, {spent_total:.1f} s of CPU work"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------------------- GPU arm

def run_sal(args, wl: synth.Workload) -> dict | None:
    import torch
    import torch.distributed as dist

    from speech_audio_encoder_b200 import api

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    B, N, L = wl.batch, wl.n_samples, wl.n_layers
    T, F = positions(N), frames(N)
    my_wl = synth.Workload(wl.name, B, N, L, wl.kind, wl.seed + rank_seed_offset(rank))
    audio = my_wl.audio()
    w = synth.make_weights(L)
    dw = api.DeviceWeights(w, device=dev)

    s = torch.cuda.Stream(device=dev)
    wave_d = torch.from_numpy(audio).to(dev)
    logmel = torch.empty((B, F, 128), dtype=torch.float32, device=dev)
    stacked = torch.empty((B, T, 1024), dtype=torch.bfloat16, device=dev)
    x = torch.empty((B * T, 1280), dtype=torch.float32, device=dev)
    emb = torch.empty((B * T, 1280), dtype=torch.bfloat16, device=dev)
    window = (api.WINDOW_CORE, api.WINDOW_CONTEXT) if args.window else None
    wcore, wctx = window if window else (0, 0)
    ws = api.encoder_workspace_ex(B, T, args.chunk, wcore, wctx, dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    lib = api.lib()
    import ctypes
    rec = ctypes.byref(dw.record)
    sp = s.cuda_stream

    opts = api.sal_forward_options(args.chunk, None, wcore, wctx)

    def step(stream_ptr=sp):
        api._check("sal_frontend", lib.sal_frontend(wave_d.data_ptr(), N, B, logmel.data_ptr(),
                                                    stacked.data_ptr(), stream_ptr))
        api._check("sal_stack_project", lib.sal_stack_project(stacked.data_ptr(), B, T, rec,
                                                              x.data_ptr(), stream_ptr))
        api._check("sal_encoder_forward_ex", lib.sal_encoder_forward_ex(
            x.data_ptr(), B, T, rec, L, emb.data_ptr(), ws.data_ptr(), ws.numel(), stream_ptr,
            ctypes.byref(opts)))

    with torch.cuda.stream(s):
        for _ in range(max(args.warmup, 3)):
            step()
    s.synchronize()
    if api.sal_last_device_status(s) != 0:
        raise RuntimeError("device wait timed out during warm-up")

    graph = torch.cuda.CUDAGraph()
    n0 = api.sal_launch_count()
    with torch.cuda.graph(graph, stream=s):
        step(torch.cuda.current_stream().cuda_stream)
    launches_per_step = api.sal_launch_count() - n0
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()

    # ---- timed region
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    gpu_id = _nvsmi_id(local)
    clocks = ClockSampler(gpu_id)
    clocks.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        for k in range(args.steps):
            flush.fill_(k & 0xFF)
            ev[k][0].record(s)
            graph.replay()
            ev[k][1].record(s)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_s = sum(step_ms) / 1e3
    total_s = reduce_max(total_s, dev)
    if api.sal_last_device_status(s) != 0:
        raise RuntimeError("device wait timed out during the timed region")
    value = job_throughput(my_wl.audio_seconds * args.steps, world, total_s)
    flops_step = workload_flops(B, T, L, args.chunk, window)

    # ---- per-kind launch durations (events around each launch, traced graph replays)
    kinds = {}
    # traced replays per kind: up to 20, fewer for long steps (about 3 s of replays per kind)
    k_steps = max(3, min(args.steps, 20, int(3000.0 / max(total_s * 1e3 / args.steps, 1e-3))))
    for kind_id, kind in enumerate(api.KIND_NAMES):
        per_step = {"rope_table": 1, "layernorm": 2 * L + 1}.get(kind, L)
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(2 * per_step)]
        for e in evs:  # torch creates the CUDA event on its first record
            e.record(s)
        s.synchronize()
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2, stream=s):
            cs = torch.cuda.current_stream().cuda_stream
            api._check("sal_frontend", lib.sal_frontend(wave_d.data_ptr(), N, B, logmel.data_ptr(),
                                                        stacked.data_ptr(), cs))
            api._check("sal_stack_project", lib.sal_stack_project(stacked.data_ptr(), B, T, rec,
                                                                  x.data_ptr(), cs))
            api.sal_encoder_forward_ex(x, B, T, dw, L, workspace=ws, emb=emb, chunk=args.chunk, kind=kind_id,
                                       events=evs, stream=cs, window_core=wcore, window_context=wctx)
        durs = []
        with torch.cuda.stream(s):
            for _ in range(k_steps):
                flush.fill_(1)
                g2.replay()
                s.synchronize()
                durs += [evs[2 * i].elapsed_time(evs[2 * i + 1]) for i in range(per_step)]
        kinds[kind] = {"launches_per_step": per_step, "avg_ms": float(np.mean(durs)),
                       "ms_per_step": float(np.mean(durs)) * per_step}
        del g2
    step_ms_mean = total_s * 1e3 / args.steps
    for k in kinds.values():
        k["share"] = k["ms_per_step"] / step_ms_mean
    tensor_kinds = ["qkv", "attention", "out_proj", "ffn_up", "ffn_down"]
    dom = max(tensor_kinds, key=lambda k: kinds[k]["ms_per_step"])
    peaks = _peaks()
    achieved = kernel_flops(dom, B, T, args.chunk, window) / (kinds[dom]["avg_ms"] / 1e3) / 1e12
    roofline = {"kernel": dom, "bound": "tensor", "achieved": achieved, "peak": peaks["tflops"],
                "unit": "TFLOP/s", "frac": achieved / peaks["tflops"],
                "traffic": _traffic(dom, wl.name) if args.chunk == 0 and not window else None,
                "peak_source": peaks["tflops_source"],
                # the same rate against the pool's sustained (power-capped) GEMM figure, and
                # the median SM clock of the timed region it ran at
                "peak_sustained": peaks["tflops_sustained"], "frac_sustained": achieved / peaks["tflops_sustained"],
                "sm_mhz_timed": clk.get("sm_mhz"),
                "per_launch_flops": kernel_flops(dom, B, T, args.chunk, window),
                "avg_launch_ms": kinds[dom]["avg_ms"]}

    # ---- the front end against HBM: algorithmic bytes (samples read once, fp32 log-mel and
    #      the bf16 stack written once) over its event-timed launch
    fe_bytes = frontend_bytes(B, N)
    # external: the records captured in the graph timestamp each replay
    fe_evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
    for e in fe_evs:
        e.record(s)
    s.synchronize()
    g3 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g3, stream=s):
        cs = torch.cuda.current_stream().cuda_stream
        fe_evs[0].record()
        api._check("sal_frontend", lib.sal_frontend(wave_d.data_ptr(), N, B, logmel.data_ptr(),
                                                    stacked.data_ptr(), cs))
        fe_evs[1].record()
    fe_ms = []
    with torch.cuda.stream(s):
        for _ in range(k_steps):
            flush.fill_(3)
            g3.replay()
            s.synchronize()
            fe_ms.append(fe_evs[0].elapsed_time(fe_evs[1]))
    del g3
    fe_avg = float(np.mean(fe_ms))
    fe_gbs = fe_bytes / (fe_avg / 1e3) / 1e9
    frontend_roofline = {"kernel": "frontend", "bound": "hbm", "achieved": fe_gbs, "peak": peaks["gbs"],
                         "unit": "GB/s", "frac": fe_gbs / peaks["gbs"], "peak_source": peaks["gbs_source"],
                         "per_launch_bytes": fe_bytes, "avg_launch_ms": fe_avg}

    # ---- end to end through sal_encode with pinned host buffers
    e2e = None
    if not args.no_e2e and args.chunk == 0 and not window:
        wave_h = torch.from_numpy(audio).pin_memory()
        emb_h = torch.empty((B, T, 1280), dtype=torch.bfloat16).pin_memory()
        ews = api.encode_workspace(B, N, dev)
        with torch.cuda.stream(s):
            for _ in range(3):
                api.sal_encode(wave_h, dw, L, emb=emb_h, workspace=ews, stream=s)
        s.synchronize()
        n_e2e = max(3, min(args.steps, 50))
        t_e2e = []
        with torch.cuda.stream(s):
            for _ in range(n_e2e):
                flush.fill_(2)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(s)
                api.sal_encode(wave_h, dw, L, emb=emb_h, workspace=ews, stream=s)
                b.record(s)
                b.synchronize()  # the result is on the host
                t_e2e.append(a.elapsed_time(b))
        e2e_s = reduce_max(sum(t_e2e) / 1e3, dev)
        e2e = {"value": job_throughput(my_wl.audio_seconds * n_e2e, world, e2e_s), "unit": UNIT,
               "h2d_bytes_per_step": B * N * 4, "d2h_bytes_per_step": B * T * 1280 * 2,
               "steps": n_e2e, "call": "sal_encode (pinned host wave in, pinned host embeddings out)"}

    # ---- oracle on the host cores (rank 0, one GPU only)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        est, desc, spent, threads = oracle_step_estimate(wl, 15.0, audio[0])
        cpu = {"value": wl.audio_seconds / est, "unit": UNIT, "cores": threads, "kind": "oracle",
               "cpu_model": _cpu_model(), "nproc": os.cpu_count(),
               "sample": desc + f"; {spent:.1f} s of CPU work"}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None
    return {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms_mean, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "batch": B, "n_samples": N, "positions": T, "layers": L,
                   "attention": (f"serving windows of {wcore} core + 2 x {wctx} context positions" if window
                                 else f"chunks of {args.chunk} positions" if 0 < args.chunk < T else "whole clip"),
                   "parallelism": f"dp{world} (independent clips per GPU)" if world > 1 else "single GPU",
                   "l2": "256 MiB buffer rewritten between timed steps", "graph": "one CUDA graph per step"},
        "tc_frac_step": flops_step / (step_ms_mean / 1e3) / 1e12 / peaks["tflops"],
        "tc_frac_step_sustained": flops_step / (step_ms_mean / 1e3) / 1e12 / peaks["tflops_sustained"],
        "roofline": roofline,
        "frontend_roofline": frontend_roofline,
        "kernels": kinds,
        "kernels_note": ("per-launch durations from event pairs around every launch of one kind in a traced "
                         "replay of the step; the event records break the programmatic-dependent-launch "
                         "overlap, so each is an upper bound and the shares need not sum to 1"),
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": int(launches_per_step * args.steps),
        "clocks": clk,
    }


def _traffic(kind: str, workload: str):
    """DRAM bytes per launch of `kind` from the committed ncu summary, or None when the
    kernel's source changed since that capture or the capture was of another workload."""
    import hashlib
    try:
        recs = json.load(open(os.path.join(ROOT, "profiles", "roofline_traffic.json")))
        rec = recs.get(f"{kind}@{workload}", recs.get(kind))
        src = open(os.path.join(ROOT, rec["source"]), "rb").read()
    except (OSError, KeyError, ValueError, TypeError, AttributeError):
        return None
    if rec.get("workload") != workload or hashlib.sha256(src).hexdigest()[:16] != rec.get("sha256_16"):
        return None
    return rec["dram_bytes_per_launch"]


def _nvsmi_id(local: int) -> str:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local < len(ids):
            return ids[local]
    return str(local)


def _peaks() -> dict:
    """Roofline denominators: the machine's measured HBM copy bandwidth and cuBLAS bf16 GEMM
    rate, burst (a kernel timed on its own) and sustained (a seconds-long loop under the
    power cap); else the fallback figures of an earlier measurement on the same pool."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        p = json.load(open(path))
        return {"tflops": float(p["bf16_tflops"]), "tflops_source": "measured (burst bf16)",
                "tflops_sustained": float(p["bf16_tflops_sustained"]),
                "gbs": float(p["hbm_gbs"]), "gbs_source": "measured"}
    except (OSError, KeyError, ValueError, TypeError):
        return {"tflops": 1590.0, "tflops_source": "fallback (burst bf16)", "tflops_sustained": 1400.0,
                "gbs": 6650.0, "gbs_source": "fallback"}


def _cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=synth.WORKLOAD_ORDER)
    ap.add_argument("--impl", default="sal", choices=["sal", "reference"])
    ap.add_argument("--chunk", type=int, default=0,
                    help="attention within chunks of this many positions (0: whole clip)")
    ap.add_argument("--window", action="store_true",
                    help="serving windows: 500 core positions with 50 context positions on each side")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.window and args.chunk:
        ap.error("--window and --chunk are exclusive")
    wl = synth.WORKLOADS[args.workload]
    out = run_reference(args, wl) if args.impl == "reference" else run_sal(args, wl)
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
