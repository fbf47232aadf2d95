#!/usr/bin/env python
"""Benchmark of the Mamba-2 mixer core on B200: prefill tokens/s and decode steps/s
with % of roofline, one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one prefill call of the whole mixer core (conv1d+SiLU, dt softplus,
chunked SSD scan, D skip, gated RMSNorm, final conv/SSM states) over the
Zamba2-2.7B-shaped workload (batch 1, 4096 tokens, 80 heads x 64, d_state 64,
bf16 I/O, fp32 state), on synthetic seeded inputs already resident in HBM.
Input/output/workspace sets rotate so that no step finds its data in the
126 MB L2.  The decode workload (batch 256, 1024 consecutive single-token
steps) is reported in the `decode` object of the same line, and the other
prefill workloads (1.2B-shaped b8 x 2048, 7B-shaped 32768-token long prefill,
the tiny fp32 case) in `workloads`, each timed the same way.

`roofline.achieved` is the path's algorithmic bytes (every input read once, y
and the final states written once) over the dominant kernel's average launch
time; `roofline.stage_bytes` is that kernel's own compulsory traffic.

Multi-GPU (torchrun, one process per GPU): every rank runs its own independent
sequence (seed = rank); there is no data-path collective (weak scaling).  The
step time is the max over ranks.

--impl reference times the fp64 CPU oracle on the same workload (a bounded
token sample per step) on this host's cores.
"""
from __future__ import annotations

import argparse
import ctypes
import itertools
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PREFILL = "zamba2_2p7b_prefill"
DECODE = "zamba2_2p7b_decode"
OTHER_PREFILL = ("zamba2_1p2b_prefill", "zamba2_7b_long_prefill", "tiny_f32")
METRIC = "SSD mixer prefill tokens/s and decode steps/s at 1 B200; % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
ROTATE = 4


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--decode-steps", type=int, default=None,
                    help="decode steps to time (default: the workload's 1024)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="time only the headline prefill workload and decode")
    return ap.parse_args()


# ---------------------------------------------------------------- accounting

def prefill_bytes(cfg) -> int:
    """Algorithmic bytes of one prefill: every input read once, y written once,
    final states written once (conv state also read when carried)."""
    e = 2 if cfg.io_dtype == "bf16" else 4
    per_token = e * (cfg.conv_dim + cfg.d_inner + cfg.nheads + cfg.d_inner)
    states = 4 * cfg.nheads * cfg.headdim * cfg.dstate + e * cfg.conv_dim * cfg.d_conv
    return cfg.batch * (cfg.seqlen * per_token + states)


def prefill_flops(cfg) -> int:
    """Algorithmic flops: causal intra-chunk (C B^T over the triangle, times X),
    chunk states, carried-state outputs; multiply-adds count 2."""
    Q, H, P, N, G = cfg.chunk_size, cfg.nheads, cfg.headdim, cfg.dstate, cfg.ngroups
    tok = cfg.batch * cfg.seqlen
    cb = G * Q * N          # C B^T, half of Q x Q x N per token pair, x2 flops
    intra = H * Q * P       # (L o CB) X over the causal triangle
    states = 2 * H * P * N  # chunk state
    off = 2 * H * P * N     # C H^T
    return tok * (cb + intra + states + off)


def decode_bytes(cfg) -> int:
    e = 2 if cfg.io_dtype == "bf16" else 4
    b = cfg.batch
    state = 2 * 4 * cfg.nheads * cfg.headdim * cfg.dstate   # read + write
    conv = 2 * e * cfg.conv_dim * cfg.d_conv               # read + write
    inputs = e * (cfg.conv_dim + cfg.d_inner + cfg.nheads)
    out = e * cfg.d_inner
    return b * (state + conv + inputs + out)


def stage_bytes(name, cfg) -> int | None:
    """Algorithmic bytes of one launch of a kernel stage: the compulsory reads of
    its inputs and writes of its outputs in their stored types."""
    e = 2 if cfg.io_dtype == "bf16" else 4
    bL = cfg.batch * cfg.seqlen
    nch = -(-cfg.seqlen // cfg.chunk_size)
    st = cfg.batch * nch * cfg.nheads * cfg.headdim * cfg.dstate * 4
    di, cd, H, GN = cfg.d_inner, cfg.conv_dim, cfg.nheads, cfg.ngroups * cfg.dstate
    table = {
        "conv_silu": bL * cd * (e + 4),
        "conv_state_out": cfg.batch * cd * cfg.d_conv * e,
        "dt_cumsum": bL * H * (e + 8),
        "chunk_state": bL * (di + GN) * 4 + bL * H * 8 + st,
        "state_pass": 2 * st + bL * H * 4 // cfg.chunk_size,
        "chunk_out": bL * cd * 4 + bL * H * 8 + st + bL * di * 4,
        "gated_norm": bL * di * (4 + e + e),
        "ssd_step": decode_bytes(cfg),
    }
    # tensor-core path (128-token chunks; u = post-conv activations, fp16;
    # S = chunk states fp32; Hc = carried states fp16; per-token dt and cumsum
    # rows fp32, written by the chunk-state kernel and read by the output kernel)
    nq = -(-cfg.seqlen // 128)
    pn = cfg.headdim * cfg.dstate
    S32 = cfg.batch * nq * H * pn * 4
    rows = 2 * cfg.batch * nq * 128 * H * 4
    table.update({
        "tc_chunk_state": bL * cd * (e + 2) + bL * H * e + S32 + cfg.batch * nq * H * 4 + rows,
        "tc_state_pass": S32 + S32 // 2 + cfg.batch * nq * H * 4 + 2 * cfg.batch * H * pn * 4,
        "tc_chunk_out": bL * (cd * 2 + di * e + di * e) + rows + S32 // 2,
    })
    return table.get(name)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d.get(k, FALLBACK_PEAKS[k])) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_hash() -> str:
    """Hash of the kernel sources: the files that define kernels and the headers
    they include (the host-only ABI code does not change what a kernel reads or
    writes, so DRAM counters taken before an edit there still hold)."""
    import hashlib
    h = hashlib.sha256()
    d = os.path.join(ROOT, "mamba_ssd_scan_mixer_b200", "csrc")
    for f in sorted(os.listdir(d)):
        with open(os.path.join(d, f), "rb") as fh:
            text = fh.read()
        if f.endswith(".cuh") or b"__global__" in text:
            h.update(f.encode() + text)
    return h.hexdigest()[:16]


def traffic_for(kernel, workload):
    """DRAM bytes per launch from a committed ncu capture, or None if there is
    none for this kernel and workload or the kernel sources changed since."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(f"{kernel}@{workload}")
    if not e or e.get("source_hash") != source_hash():
        return None
    return e.get("bytes_per_launch")


# ---------------------------------------------------------------- ranks

def rank_seed(rank: int) -> int:
    """Each rank runs its own independent sequence (weak scaling)."""
    return rank


def max_over_ranks(value: float, world: int, device) -> float:
    """The slowest rank's time: all-reduce MAX (every rank must call this)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank_step: int, steps: int, max_elapsed_ms: float, world: int) -> float:
    """Whole-job throughput: units all ranks processed / the slowest rank's time."""
    return world * units_per_rank_step * steps / (max_elapsed_ms / 1e3)


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.proc = None
        self.gpu = gpu_index
        self.path = f"/tmp/m2bench_clocks_{os.getpid()}.csv"

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.fh,
                stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        pw = [num(r[3]) for r in rows if num(r[3]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        busy = [s for s, p in zip(sm, pw) if p is not None and p > 200] or sm
        return {"sm_mhz": statistics.median(busy) if busy else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(pw) if pw else None}


# ---------------------------------------------------------------- our arm

def kernel_chunk(cfg, stage_names) -> int:
    """Chunk length the kernels of this call really use: the tensor-core path
    (its stages are named tc_*) always runs 128-token chunks, the CUDA-core path
    honours the configured chunk_size."""
    return 128 if any(n.startswith("tc_") for n in stage_names) else cfg.chunk_size


def measure_prefill(name, args, dev, stream, seed, world, peaks, peak_src, m2, W, lib,
                    steps=None, warmup=None, flush_l2=False):
    """Device-timed prefill steps of workload `name` (inputs resident in HBM).

    Input/output/workspace sets rotate so that a step never finds its data in
    L2 (the rotation's total exceeds the 126 MB L2); with flush_l2 (for
    workloads too small for that) a 256 MB buffer is written between steps and
    each step is timed on its own.  Every stage is bracketed once per warm-up
    step; the dominant one is then bracketed by its own events in every timed
    step."""
    import torch
    import torch.distributed as dist
    cfg = W.CONFIGS[name]
    dims = m2.dims_from_config(cfg)
    params = {k: v.to(dev) for k, v in W.make_params(cfg, seed).items()}
    pp = m2.make_params(params["conv_w"], params["conv_b"], params["dt_bias"], params["A"],
                        params["D"], params["norm_w"])
    host_in = W.make_prefill_inputs(cfg, seed)["zxbcdt"]
    di, cd = cfg.d_inner, cfg.conv_dim
    ws_bytes = m2.mamba2_prefill_workspace_size(dims)
    in_bytes = host_in.numel() * host_in.element_size()
    rotate = 1 if flush_l2 else max(2, min(ROTATE, -(-4 * 126_000_000 // max(1, in_bytes))))
    sets = []
    for r in range(rotate):
        packed = host_in.to(dev)
        v = W.split_packed(cfg, packed)
        sets.append(dict(
            packed=packed, z=v["z"], xBC=v["xBC"], dt=v["dt_raw"],
            y=torch.empty(cfg.batch, cfg.seqlen, di, dtype=cfg.torch_dtype, device=dev),
            cs=torch.zeros(cfg.batch, cd, cfg.d_conv, dtype=cfg.torch_dtype, device=dev),
            hs=torch.zeros(cfg.batch, cfg.nheads, cfg.headdim, cfg.dstate, device=dev),
            ws=torch.empty(max(1, ws_bytes), dtype=torch.uint8, device=dev)))
    rot_bytes = sum(sum(t.numel() * t.element_size() for k, t in s.items()
                        if k in ("packed", "y", "cs", "hs", "ws")) for s in sets)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev) if flush_l2 else None

    names_arr = (ctypes.c_char_p * 16)()
    nst = lib.mamba2_stage_names(0, ctypes.byref(dims), names_arr, 16)
    stage_names = [names_arr[i].decode() for i in range(nst)]

    def call(s, events=None):
        if events is not None:
            arr = (ctypes.c_void_p * len(events))(*events)
            lib.mamba2_record_stage_events(arr, len(events))
        m2.mamba2_conv_ssd_prefill(dims, pp, s["xBC"], s["z"], s["dt"], s["y"], s["cs"],
                                   s["hs"], False, s["ws"], stream)

    def new_event():
        e = torch.cuda.Event(enable_timing=True)
        e.record(stream)
        return e

    W_ = max(3, args.warmup if warmup is None else warmup)
    stage_ms = [0.0] * nst
    n_stage = 0
    for i in range(W_):
        if flush is not None:
            flush.fill_(i & 255)
        evs = [new_event() for _ in range(nst + 1)]
        call(sets[i % rotate], [e.cuda_event for e in evs])
        torch.cuda.synchronize(dev)
        if i >= min(2, W_ - 1):  # the first calls pay one-time costs: not counted
            n_stage += 1
            for j in range(nst):
                stage_ms[j] += evs[j].elapsed_time(evs[j + 1])
    dom = max(range(nst), key=lambda j: stage_ms[j])

    K = args.steps if steps is None else steps
    dom_evs = [(new_event(), new_event()) for _ in range(K)]
    step_evs = [(new_event(), new_event()) for _ in range(K)] if flush is not None else None
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for k in range(K):
        if flush is not None:
            flush.fill_(k & 255)
            step_evs[k][0].record(stream)
        a, b = dom_evs[k]
        call(sets[k % rotate], [None] * dom + [a.cuda_event, b.cuda_event])
        if flush is not None:
            step_evs[k][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    elapsed = (sum(a.elapsed_time(b) for a, b in step_evs) if flush is not None
               else t0.elapsed_time(t1))
    dom_ms = sum(a.elapsed_time(b) for a, b in dom_evs) / K
    elapsed = max_over_ranks(elapsed, world, dev)
    ms = elapsed / K
    tokens = cfg.batch * cfg.seqlen
    path_bytes = prefill_bytes(cfg)
    path_flops = prefill_flops(cfg)
    t_roof = max(path_bytes / (peaks["hbm_gbs"] * 1e9),
                 path_flops / (peaks["bf16_tflops"] * 1e12))
    dom_name = stage_names[dom]
    achieved = path_bytes / (dom_ms * 1e-3) / 1e9
    sbytes = stage_bytes(dom_name, cfg)
    out = {
        "value": job_rate(tokens, K, elapsed, world), "unit": "tokens/s", "steps": K,
        "warmup": W_, "ms_per_step": ms,
        "config": {"workload": name, "batch": cfg.batch, "seqlen": cfg.seqlen,
                   "nheads": cfg.nheads, "headdim": cfg.headdim, "dstate": cfg.dstate,
                   "ngroups": cfg.ngroups, "io_dtype": cfg.io_dtype,
                   "chunk": kernel_chunk(cfg, stage_names),
                   "chunk_size_setting": cfg.chunk_size, "state_dtype": "f32",
                   "l2": (f"L2 flushed (256 MB write) before every step, steps timed one by one"
                          if flush is not None else
                          f"{rotate} rotating input/output/workspace sets, "
                          f"{rot_bytes / 1e9:.2f} GB > 126 MB L2")},
        # achieved = the path's algorithmic bytes (every input read once, y and the
        # final states written once) over the dominant kernel's average launch time
        "roofline": {"bound": "hbm", "kernel": dom_name, "achieved": achieved,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"],
                     "traffic": traffic_for(dom_name, name),
                     "algorithmic_bytes": path_bytes, "avg_launch_ms": dom_ms,
                     "stage_bytes": sbytes,
                     "stage_gbs": sbytes / (dom_ms * 1e-3) / 1e9 if sbytes else None,
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)"
                     if peak_src == "measured" else "fallback 6650 GB/s"},
        "path_roofline": {"bytes": path_bytes, "flops": path_flops,
                          "roofline_ms": t_roof * 1e3,
                          "achieved_gbs": path_bytes / (ms * 1e-3) / 1e9,
                          "frac": t_roof * 1e3 / ms, "peak_source": peak_src},
        "stages_ms_warmup_avg": {n: stage_ms[j] / n_stage for j, n in enumerate(stage_names)},
        "gpu_launches": K * nst,
    }
    del sets, flush
    torch.cuda.empty_cache()
    return out


# Packed-sequence prefill: eight requests of mixed lengths (4096 tokens in all,
# from a single token to 1600, with chunk tails and an exact multiple of 128)
# on the 2.7B-shaped mixer, each continuing from its own carried state.
VARLEN_LENGTHS = (1, 3, 127, 129, 512, 700, 1024, 1600)


def measure_backward(args, dev, stream, seed, world, peaks, peak_src, m2, W, lib, steps, warmup):
    """Device-timed backward passes of the 2.7B prefill (mamba2_conv_ssd_prefill_backward:
    forward recomputed, all gradients), carried states in and a final-state gradient,
    steps timed one by one (each call writes and reads GBs: far beyond L2)."""
    import torch
    cfg = W.CONFIGS[PREFILL]
    dims = m2.dims_from_config(cfg)
    params = {k: v.to(dev) for k, v in W.make_params(cfg, seed).items()}
    pp = m2.make_params(params["conv_w"], params["conv_b"], params["dt_bias"], params["A"],
                        params["D"], params["norm_w"])
    v = W.split_packed(cfg, W.make_prefill_inputs(cfg, seed)["zxbcdt"].to(dev))
    st = W.make_states(cfg, seed)
    cs, hs = st["conv_state"].to(dev), st["ssm_state"].to(dev)
    g = torch.Generator(device=dev).manual_seed(2000 + seed)
    dy = torch.randn(cfg.batch, cfg.seqlen, cfg.d_inner, generator=g, device=dev).to(
        cfg.torch_dtype)
    dhl = 0.1 * torch.randn(hs.shape, generator=g, device=dev)
    ws = torch.empty(max(1, m2.mamba2_prefill_backward_workspace_size(dims)), dtype=torch.uint8,
                     device=dev)
    names_arr = (ctypes.c_char_p * 16)()
    nst = lib.mamba2_stage_names(2, ctypes.byref(dims), names_arr, 16)
    stage_names = [names_arr[i].decode() for i in range(nst)]
    grads = None

    def call(stage_events=None):
        nonlocal grads
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        if stage_events is not None:
            arr = (ctypes.c_void_p * len(stage_events))(*[e.cuda_event for e in stage_events])
            lib.mamba2_record_stage_events(arr, len(stage_events))
        grads = m2.prefill_backward(dims, pp, v["xBC"], v["z"], v["dt_raw"], dy, cs, hs, dhl,
                                    ws, stream)
        b.record(stream)
        return a, b

    stage_ms, n_stage = [0.0] * nst, 0
    for i in range(max(3, warmup)):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)]
        for ev in evs:
            ev.record(stream)
        call(evs)
        torch.cuda.synchronize(dev)
        if i >= 2:
            n_stage += 1
            for j in range(nst):
                stage_ms[j] += evs[j].elapsed_time(evs[j + 1])
    evs = [call() for _ in range(steps)]
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), world, dev) / steps
    T, e = cfg.batch * cfg.seqlen, 2
    # compulsory bytes: the forward's inputs and dy read, the input gradients written
    # (bf16); the states and their gradients (fp32 SSM, bf16 conv) read / written once
    states = 4 * cfg.nheads * cfg.headdim * cfg.dstate + e * cfg.conv_dim * cfg.d_conv
    io = cfg.conv_dim + cfg.d_inner + cfg.nheads
    path_bytes = T * e * (io + cfg.d_inner + io) + cfg.batch * 3 * states
    t_roof = path_bytes / (peaks["hbm_gbs"] * 1e9)
    return {
        "value": job_rate(T, steps, ms * steps, world), "unit": "tokens/s", "steps": steps,
        "warmup": max(3, warmup), "ms_per_step": ms,
        "config": {"workload": "zamba2_2p7b_prefill_backward", "batch": cfg.batch,
                   "seqlen": cfg.seqlen, "nheads": cfg.nheads, "headdim": cfg.headdim,
                   "dstate": cfg.dstate, "ngroups": cfg.ngroups, "io_dtype": cfg.io_dtype,
                   "compute": "fp32 CUDA cores", "states_in": True,
                   "workspace_bytes": ws.numel(),
                   "l2": "each call writes and reads the per-token states (GBs)"},
        "path_roofline": {"bytes": path_bytes, "roofline_ms": t_roof * 1e3,
                          "achieved_gbs": path_bytes / (ms * 1e-3) / 1e9,
                          "frac": t_roof * 1e3 / ms, "peak_source": peak_src},
        "stages_ms_warmup_avg": {n: stage_ms[j] / max(1, n_stage)
                                 for j, n in enumerate(stage_names)},
        "gpu_launches": 9 * steps,
    }


def measure_varlen(args, dev, stream, seed, world, peaks, peak_src, m2, W, lib, steps, warmup):
    """Device-timed packed-sequence prefills (mamba2_conv_ssd_prefill_varlen), L2
    flushed (256 MB write) before every step, steps timed one by one."""
    import torch
    T, n = sum(VARLEN_LENGTHS), len(VARLEN_LENGTHS)
    cfg1 = W.CONFIGS[PREFILL].with_(batch=1, seqlen=T)
    cfg = cfg1.with_(batch=n)  # dims: batch = sequences, seqlen = total tokens
    dims = m2.dims_from_config(cfg)
    params = {k: v.to(dev) for k, v in W.make_params(cfg, seed).items()}
    pp = m2.make_params(params["conv_w"], params["conv_b"], params["dt_bias"], params["A"],
                        params["D"], params["norm_w"])
    v = W.split_packed(cfg1, W.make_prefill_inputs(cfg1, seed)["zxbcdt"][0].to(dev))
    st = W.make_states(cfg, seed)
    cs0, hs0 = st["conv_state"].to(dev), st["ssm_state"].to(dev)
    cs, hs = cs0.clone(), hs0.clone()
    cu = torch.tensor([0] + list(itertools.accumulate(VARLEN_LENGTHS)), dtype=torch.int32,
                      device=dev)
    y = torch.empty(T, cfg.d_inner, dtype=cfg.torch_dtype, device=dev)
    ws = torch.empty(max(1, m2.mamba2_prefill_varlen_workspace_size(dims)), dtype=torch.uint8,
                     device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    names_arr = (ctypes.c_char_p * 16)()
    nst = lib.mamba2_stage_names(0, ctypes.byref(dims), names_arr, 16)
    stage_names = [names_arr[i].decode() for i in range(nst)]

    def call(stage_events=None):
        cs.copy_(cs0)  # every step continues from the same carried states
        hs.copy_(hs0)
        flush.fill_(1)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        if stage_events is not None:
            arr = (ctypes.c_void_p * len(stage_events))(*[e.cuda_event for e in stage_events])
            lib.mamba2_record_stage_events(arr, len(stage_events))
        m2.mamba2_conv_ssd_prefill_varlen(dims, pp, v["xBC"], v["z"], v["dt_raw"], cu, y, cs, hs,
                                          True, ws, stream)
        b.record(stream)
        return a, b

    stage_ms, n_stage = [0.0] * nst, 0
    for i in range(max(3, warmup)):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)]
        for ev in evs:
            ev.record(stream)  # torch creates the CUDA event on its first record
        call(evs)
        torch.cuda.synchronize(dev)
        if i >= 2:  # the first calls pay one-time costs
            n_stage += 1
            for j in range(nst):
                stage_ms[j] += evs[j].elapsed_time(evs[j + 1])
    torch.cuda.synchronize(dev)
    evs = [call() for _ in range(steps)]
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), world, dev) / steps
    e = 2
    states = 4 * cfg.nheads * cfg.headdim * cfg.dstate + e * cfg.conv_dim * cfg.d_conv
    path_bytes = T * e * (cfg.conv_dim + 2 * cfg.d_inner + cfg.nheads) + n * 2 * states
    path_flops = prefill_flops(cfg1)
    t_roof = max(path_bytes / (peaks["hbm_gbs"] * 1e9), path_flops / (peaks["bf16_tflops"] * 1e12))
    return {
        "value": job_rate(T, steps, ms * steps, world), "unit": "tokens/s", "steps": steps,
        "warmup": max(3, warmup), "ms_per_step": ms,
        "config": {"workload": "zamba2_2p7b_varlen_prefill", "sequences": n,
                   "lengths": list(VARLEN_LENGTHS), "tokens": T, "nheads": cfg.nheads,
                   "headdim": cfg.headdim, "dstate": cfg.dstate, "ngroups": cfg.ngroups,
                   "io_dtype": cfg.io_dtype, "chunk": 128, "states_in": True,
                   "l2": "L2 flushed (256 MB write) before every step, steps timed one by one"},
        # every input and carried state read once, y and the final states written once
        "path_roofline": {"bytes": path_bytes, "flops": path_flops,
                          "roofline_ms": t_roof * 1e3,
                          "achieved_gbs": path_bytes / (ms * 1e-3) / 1e9,
                          "frac": t_roof * 1e3 / ms, "peak_source": peak_src},
        # (the first stage includes the small kernel that lays out the chunks)
        "stages_ms_warmup_avg": {n: stage_ms[j] / max(1, n_stage)
                                 for j, n in enumerate(stage_names)},
        "gpu_launches": 4 * steps,
    }


def run_ours(args, rank, world, local_rank):
    import torch
    import mamba_ssd_scan_mixer_b200 as m2
    from mamba_ssd_scan_mixer_b200 import workloads as W

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = W.CONFIGS[PREFILL]
    seed = rank_seed(rank)
    lib = m2.lib()
    dims = m2.dims_from_config(cfg)
    stream = torch.cuda.current_stream(dev)
    peaks, peak_src = load_peaks()

    sampler = ClockSampler(local_rank) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    head = measure_prefill(PREFILL, args, dev, stream, seed, world, peaks, peak_src, m2, W, lib)
    clocks = sampler.stop() if sampler else None

    line = {
        "metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": head["steps"], "warmup": head["warmup"], "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": dict(head["config"], parallelism=f"dp{world} (independent sequences)"),
        "roofline": head["roofline"], "path_roofline": head["path_roofline"],
        "stages_ms_warmup_avg": head["stages_ms_warmup_avg"],
        "gpu_launches": head["gpu_launches"], "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_e2e:
        line["e2e"] = run_e2e(args, cfg, dims, head_params(cfg, seed, dev, m2, W),
                              W.make_prefill_inputs(cfg, seed)["zxbcdt"], dev, stream, m2)
    if not args.no_decode:
        line["decode"] = run_decode(args, dev, stream, rank, world, peaks, peak_src, m2, W)
        line["gpu_launches"] += line["decode"]["gpu_launches"]
    if not args.no_workloads:
        # the other prefill workloads: parity-tested shapes, timed the same way
        other = {}
        for name in OTHER_PREFILL:
            small = W.CONFIGS[name].batch * W.CONFIGS[name].seqlen < 65536
            o = measure_prefill(name, args, dev, stream, seed, world, peaks, peak_src, m2, W,
                                lib, steps=min(args.steps, 20), warmup=3, flush_l2=small)
            line["gpu_launches"] += o.pop("gpu_launches")
            other[name] = o
        o = measure_varlen(args, dev, stream, seed, world, peaks, peak_src, m2, W, lib,
                           steps=min(args.steps, 20), warmup=3)
        line["gpu_launches"] += o.pop("gpu_launches")
        other["zamba2_2p7b_varlen_prefill"] = o
        o = measure_backward(args, dev, stream, seed, world, peaks, peak_src, m2, W, lib,
                             steps=min(args.steps, 5), warmup=3)
        line["gpu_launches"] += o.pop("gpu_launches")
        other["zamba2_2p7b_prefill_backward"] = o
        line["workloads"] = other
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, seconds=10.0)
    return line


def head_params(cfg, seed, dev, m2, W):
    params = {k: v.to(dev) for k, v in W.make_params(cfg, seed).items()}
    pp = m2.make_params(params["conv_w"], params["conv_b"], params["dt_bias"], params["A"],
                        params["D"], params["norm_w"])
    pp._keep = params  # the tensors must outlive the pointers
    return pp


def run_e2e(args, cfg, dims, pp, host_in, dev, stream, m2):
    """Tokens/s through the host-buffer entry point (mamba2_conv_ssd_prefill_host):
    each step's inputs start in page-locked host memory and its y and final states
    end there; the library overlaps the copies with the work, piece by piece."""
    import torch
    from mamba_ssd_scan_mixer_b200 import workloads as W
    di, cd = cfg.d_inner, cfg.conv_dim
    h_in = host_in.pin_memory()
    h_y = torch.empty(cfg.batch, cfg.seqlen, di, dtype=cfg.torch_dtype).pin_memory()
    h_cs = torch.empty(cfg.batch, cd, cfg.d_conv, dtype=cfg.torch_dtype).pin_memory()
    h_hs = torch.empty(cfg.batch, cfg.nheads, cfg.headdim, cfg.dstate).pin_memory()
    ws = torch.empty(max(1, m2.mamba2_prefill_host_workspace_size(dims)), dtype=torch.uint8,
                     device=dev)
    v = W.split_packed(cfg, h_in)

    def step():
        m2.mamba2_conv_ssd_prefill_host(dims, pp, v["xBC"], v["z"], v["dt_raw"], h_y, h_cs, h_hs,
                                        False, ws, stream)

    for _ in range(3):
        step()
    torch.cuda.synchronize(dev)
    K = max(3, min(args.steps, 50))
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(K):
        step()
    b.record(stream)
    torch.cuda.synchronize(dev)
    ms = a.elapsed_time(b) / K
    nbytes = lambda t: t.numel() * t.element_size()
    h2d = cfg.batch * cfg.seqlen * (cd + di + cfg.nheads) * h_in.element_size()
    return {"value": cfg.batch * cfg.seqlen / (ms * 1e-3), "unit": "tokens/s", "steps": K,
            "ms_per_step": ms, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": nbytes(h_y) + nbytes(h_cs) + nbytes(h_hs),
            "entry": "mamba2_conv_ssd_prefill_host (pieces of whole chunks, copies overlapped)"}


def run_decode(args, dev, stream, rank, world, peaks, peak_src, m2, W):
    """The batch-256 decode workload: consecutive single-token steps with distinct
    per-step inputs (pre-generated on the device), states updated in place."""
    import torch
    import torch.distributed as dist
    cfg = W.CONFIGS[DECODE]
    S = args.decode_steps or cfg.decode_steps
    dims = m2.dims_from_config(cfg)
    params = {k: v.to(dev) for k, v in W.make_params(cfg, rank_seed(rank)).items()}
    pp = m2.make_params(params["conv_w"], params["conv_b"], params["dt_bias"], params["A"],
                        params["D"], params["norm_w"])
    st = W.make_states(cfg, rank_seed(rank))
    cs = st["conv_state"].to(dev)
    hs = st["ssm_state"].to(dev)
    g = torch.Generator(device=dev).manual_seed(1000 + rank)
    inputs = torch.randn(S, cfg.batch, cfg.packed_width, generator=g, device=dev).to(
        cfg.torch_dtype)
    y = torch.empty(cfg.batch, cfg.d_inner, dtype=cfg.torch_dtype, device=dev)
    di, cd = cfg.d_inner, cfg.conv_dim

    def step(k):
        v = W.split_packed(cfg, inputs[k])
        m2.mamba2_ssd_step(dims, pp, v["xBC"], v["z"], v["dt_raw"], y, cs, hs, stream)

    for k in range(max(3, args.warmup)):
        step(k % S)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(dev.index) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for k in range(S):
        step(k)
    b.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    elapsed = a.elapsed_time(b)
    clocks = sampler.stop() if sampler else None
    elapsed = max_over_ranks(elapsed, world, dev)
    ms = elapsed / S
    nb = decode_bytes(cfg)
    ach = nb / (ms * 1e-3) / 1e9
    return {"value": job_rate(1, S, elapsed, world), "unit": "steps/s", "steps": S,
            "ms_per_step": ms, "tokens_per_s": job_rate(cfg.batch, S, elapsed, world),
            "config": {"workload": DECODE, "batch": cfg.batch, "nheads": cfg.nheads,
                       "headdim": cfg.headdim, "dstate": cfg.dstate,
                       "l2": "state 335 MB > 126 MB L2; distinct per-step inputs"},
            "roofline": {"bound": "hbm", "kernel": "ssd_step", "achieved": ach,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": ach / peaks["hbm_gbs"], "traffic": traffic_for("ssd_step", DECODE),
                         "algorithmic_bytes": nb, "peak_source": peak_src},
            "gpu_launches": S, "clocks": clocks}


# ---------------------------------------------------------------- CPU oracle

def _oracle_tokens(cfg, params, inp, ntok, nthreads):
    import oracle
    t = time.perf_counter()
    oracle.mixer_prefill(inp["xBC"][:, :ntok], inp["z"][:, :ntok], inp["dt_raw"][:, :ntok],
                         params, nheads=cfg.nheads, headdim=cfg.headdim, dstate=cfg.dstate,
                         ngroups=cfg.ngroups, eps=cfg.norm_eps,
                         norm_before_gate=cfg.norm_before_gate, nthreads=nthreads)
    return time.perf_counter() - t


def cpu_baseline(cfg, seconds=10.0):
    """The fp64 oracle, as it stands, on the prefill workload: whole 4096-token
    passes repeated until `seconds` of CPU time have run (at least one)."""
    import oracle
    from mamba_ssd_scan_mixer_b200 import workloads as W
    params = W.make_params(cfg, 0)
    inp = W.make_prefill_inputs(cfg, 0)
    cores = oracle.default_threads()
    total_t, runs = 0.0, 0
    while runs == 0 or (total_t < seconds and runs < 20):
        total_t += _oracle_tokens(cfg, params, inp, cfg.seqlen, cores)
        runs += 1
    return {"value": runs * cfg.batch * cfg.seqlen / total_t, "unit": "tokens/s",
            "cores": cores, "kind": "oracle",
            "sample": f"{runs} full pass(es) of the {PREFILL} workload "
                      f"({cfg.batch}x{cfg.seqlen} tokens, all {cfg.nheads} heads), "
                      f"{total_t:.1f} s"}


def run_reference(args):
    """Reference arm: the fp64 CPU oracle on the same workload and metric, each
    step a bounded prefix of the 4096-token sequence (all heads)."""
    from mamba_ssd_scan_mixer_b200 import workloads as W
    import oracle
    cfg = W.CONFIGS[PREFILL]
    params = W.make_params(cfg, 0)
    inp = W.make_prefill_inputs(cfg, 0)
    cores = oracle.default_threads()
    # size each step so that warm-up + steps take about 90 s in total
    calib = 256
    t_tok = _oracle_tokens(cfg, params, inp, calib, cores) / calib
    K, Wm = args.steps, max(3, args.warmup)
    ntok = int(max(16, min(cfg.seqlen, 90.0 / max(1, K + Wm) / max(t_tok, 1e-9))))
    for _ in range(Wm):
        _oracle_tokens(cfg, params, inp, ntok, cores)
    total = sum(_oracle_tokens(cfg, params, inp, ntok, cores) for _ in range(K))
    value = K * cfg.batch * ntok / total
    return {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": K, "warmup": Wm, "ms_per_step": total / K * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": PREFILL, "batch": cfg.batch, "seqlen": cfg.seqlen,
                       "nheads": cfg.nheads, "headdim": cfg.headdim, "dstate": cfg.dstate,
                       "ngroups": cfg.ngroups, "chunk": cfg.chunk_size},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                             "kind": "oracle",
                             "sample": f"first {ntok} of {cfg.seqlen} tokens per step, "
                                       f"all {cfg.nheads} heads"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0
    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
